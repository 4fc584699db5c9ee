/*
 * emp.h -- C ABI of the B200 equivariant edge message-passing library.
 *
 * The library computes the per-edge equivariant SO(2) message-passing
 * convolution of a machine-learned interatomic potential (lmax = 3) and its
 * input-gradient (force) backward, as described on the page "deepmd-kit PR:
 * first-order SO(2) input-gradient path" (sections "Implementation and scope"
 * and "Multi-model and N4096 update": 8192-edge receiver-sorted cohorts, strict
 * FP32), with the radial projection chain of the page "deepmd-kit PR #6108:
 * radial head fold" (section "What").
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless the comment says (host).
 *   - The caller owns every input, output and workspace buffer.  The library
 *     owns only the model / chain objects it creates.  Inputs are never
 *     written; outputs must not alias inputs.  (Ownership rule of the page
 *     "first-order SO(2) input-gradient path", section "Implementation and
 *     scope": never overwrite caller inputs.)
 *   - Every call enqueues work on `stream` and returns; the only host
 *     synchronisation is nl_build's read-back of the edge count.
 *   - Results are bitwise identical from run to run (no floating-point
 *     atomics; every sum has a fixed order).
 *   - Errors are returned as emp_status codes; no exception crosses the ABI.
 *     Errors detected on the device (index out of range, a bounded wait that
 *     ran out) set a device error word reported by emp_last_device_error().
 *
 * Layouts
 *   positions     double [N][3]
 *   node features float  [N][16][C], component index lm = l*l + l + m
 *                 (m = -l..l), channel-contiguous; real orthonormal spherical
 *                 harmonics with z as polar axis, no Condon-Shortley phase
 *                 (degree 1 is ordered y, z, x)
 *   edges         sorted by receiver, then sender, then image shift
 */
#ifndef EMP_H
#define EMP_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  EMP_OK = 0,
  EMP_ERR_ARG = -1,        /* null pointer, bad size or alignment, inconsistent spec */
  EMP_ERR_CAPACITY = -2,   /* graph buffers smaller than the edge count (see nl_build) */
  EMP_ERR_CUDA = -3,       /* a CUDA runtime call failed */
  EMP_ERR_TIMEOUT = -4,    /* a bounded device wait gave up */
  EMP_ERR_NONFINITE = -5,  /* non-finite positions */
  EMP_ERR_WORKSPACE = -6,  /* workspace smaller than the *_workspace_bytes value */
  EMP_ERR_DEVICE = -7,     /* device-side check failed (index out of range, degree limit) */
  EMP_ERR_UNSUPPORTED = -8 /* no sm_100 device, or a size the kernels do not support */
} emp_status;

/* ------------------------------------------------------------ neighbour list
 * Defined on the page "first-order SO(2) input-gradient path" only as "the
 * neighbour list" of the N64 / N4096 diamond workloads; this library builds
 * the bit-exact cell-list form: an edge (i, j, S) exists iff, with
 * r = (x_j - x_i) + S * L per Cartesian component in IEEE double (separate
 * roundings, no fused multiply-add) and d2 = (rx*rx + ry*ry) + rz*rz,
 * d2 < cutoff*cutoff; (i, i, 0) is excluded.  i is the receiver, j the sender.
 */
typedef struct {
  int32_t n_atoms;
  double box[3];       /* orthorhombic periodic box edges L (angstrom) */
  double cutoff;       /* rc (angstrom) */
  int64_t capacity;    /* edge capacity of the graph buffers */
} emp_nl_params;

typedef struct {
  int32_t* recv;       /* [capacity] receiver i */
  int32_t* send;       /* [capacity] sender j */
  int32_t* mirror;     /* [capacity] index of the edge (j, i, -S) */
  int32_t* recv_off;   /* [N+1] CSR offsets over receivers */
  int32_t* shift;      /* [capacity][3] image shift S */
  float* vec;          /* [capacity][3] r rounded to float32 */
  int64_t n_edges;     /* number of valid edges (set by nl_build); with 0 edges the
                          per-edge pointers may be NULL in the mp_* calls */
  int32_t n_atoms;     /* number of atoms N (set by nl_build) */
} emp_graph;

/* Workspace bytes nl_build needs for n_atoms atoms. */
size_t nl_workspace_bytes(int32_t n_atoms);

/* Build the neighbour list of `pos` into `g`.
 * n_edges (host, out): the edge count, set also when EMP_ERR_CAPACITY is
 * returned (two-phase use: call once with capacity 0 to size the buffers).
 * Errors: EMP_ERR_ARG (null pointers, n_atoms < 1, non-positive box or
 * cutoff), EMP_ERR_NONFINITE, EMP_ERR_CAPACITY, EMP_ERR_WORKSPACE,
 * EMP_ERR_DEVICE (a receiver with more than 4096 neighbours),
 * EMP_ERR_UNSUPPORTED (an edge whose image shift has a component beyond
 * +-127 box lengths, e.g. unwrapped positions that drifted that far apart).
 * On these two the edge count is still reported and the graph is not written. */
int nl_build(const emp_nl_params* p, const double* pos, emp_graph* g, int64_t* n_edges,
             void* ws, size_t ws_bytes, cudaStream_t stream);

/* Same neighbour list as nl_build, for callers that cannot allocate device
 * memory (for example a plug-in inside a host program that owns all device
 * memory through its own pool, or a code path that must not trigger the
 * device-wide synchronisation that cudaMalloc / cudaFree can cause).  The
 * caller still provides positions and the graph buffers; the cell-list scratch
 * is a fixed array inside the library (EMP_NL_NOALLOC_SCRATCH_BYTES, held by
 * every device that loads the library until the process exits).  Nothing is
 * allocated.  The subject pages have no counterpart of this entry point.
 *   - n_atoms above EMP_NL_NOALLOC_MAX_ATOMS: EMP_ERR_WORKSPACE.
 *   - Each call looks up the scratch array's device address on the current
 *     device (cudaGetSymbolAddress); make the first call on a device before
 *     any stream capture (it loads the library's module on that device).
 *   - All calls on a device share the scratch; calls whose GPU work overlaps
 *     (unordered streams) race on it.  Each call clears what must start at zero.
 * Other arguments, results and errors as nl_build. */
#define EMP_NL_NOALLOC_MAX_ATOMS 65536
#define EMP_NL_NOALLOC_SCRATCH_BYTES (3u << 20)
int nl_build_noalloc(const emp_nl_params* p, const double* pos, emp_graph* g, int64_t* n_edges,
                     cudaStream_t stream);

/* Neighbour-list reuse in an MD loop (skin).  A graph built by nl_build with cutoff
 * rc + skin at positions pos_ref stays valid for a model of cutoff rc while no atom has
 * moved more than skin / 2: the edges longer than rc contribute exactly zero (the radial
 * envelope and its derivative vanish there and every layer is bias-free).  nl_refresh
 * writes the edge vectors of g at the new positions pos (same edges and shifts, the same
 * double-precision operations as nl_build, rounded to float) and sets rebuild (host, out)
 * to 1 when some atom is more than skin / 2 from its pos_ref position (then call nl_build
 * again), else 0.  p: the box and n_atoms of the build.  Workspace >= 64 bytes.
 * Synchronises (reads the displacement back).  Errors: EMP_ERR_ARG, EMP_ERR_NONFINITE. */
int nl_refresh(const emp_nl_params* p, const double* pos, const double* pos_ref, double skin, emp_graph* g,
               int32_t* rebuild, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ the model
 * Hyper-parameters of the interatomic potential (configs of the seeded
 * workloads; model of the page "first-order SO(2) input-gradient path":
 * lmax = 3, three layers, strict FP32).  lmax is fixed at 3. */
typedef struct {
  int32_t C;              /* channels per component; multiple of 32, 32..256 */
  int32_t n_layers;       /* interaction layers (>= 1) */
  int32_t n_species;      /* >= 1 */
  int32_t n_basis;        /* Bessel functions; must be 8 */
  int32_t radial_hidden;  /* radial MLP width; must be 64 */
  int32_t readout_hidden; /* readout MLP width (<= 256) */
  int32_t gated;          /* 1: x <- x + G(agg) after each layer; 0: h = agg */
  int32_t pair_radial;    /* 1: one radial MLP per unordered species pair */
  int32_t cohort_edges;   /* receiver-sorted edge cohort size (multiple of 128, <= 16384) */
  float cutoff;           /* rc */
  int32_t env_p;          /* envelope exponent; must be 6 */
  float avg_degree;       /* aggregation normaliser (158) */
} emp_model_spec;

/* Number of floats of the weight blob for `spec` (declaration order: emb
 * [S][C]; per layer: per radial network W1 [H][8], W2 [H][H], W3 [4C][H];
 * W0 [4C][4C]; for m = 1, 2, 3: Wr_m, Wi_m [(4-m)C][(4-m)C]; then readout
 * W_ro [H_ro][C], w_o [H_ro]).  All linear maps bias-free, stored (out, in). */
size_t mp_weight_count(const emp_model_spec* spec);

/* Copy (host blob -> device), stack the SO(2) blocks, split them for
 * 3xTF32 and build the rotation generators.  model (host, out). */
int mp_model_create(const emp_model_spec* spec, const float* weights /*(host)*/, size_t n_floats,
                    void** model);
void mp_model_destroy(void* model);

/* Certified radial tables (opt-in approximation; page FastMACE, "Rewrite screens:
 * adopted and rejected", OPT6-T04 / OPT6-T05 radial tables).  With tol > 0, builds for
 * every layer and radial network, in double precision on the host, a piecewise Chebyshev
 * table of degree 10 of the network's hidden output h2(d) (64 values) on dyadic pieces of
 * [0, cutoff], bisected until every value and length derivative is within tol of its local
 * scale (its largest magnitude on the piece, at least 1e-3 of its largest magnitude on
 * [0, cutoff]); from then on mp_forward and mp_energy_forces evaluate h2 and its length
 * derivative from the tables (float32, on the device) instead of the network's hidden
 * layers; the head W3 stays a product.  tol <= 0 frees the tables and goes back to the
 * network.  The model owns the tables.  n_pieces (host, out, may be NULL): pieces over all
 * tables.  Synchronous.  Errors: EMP_ERR_ARG (no model, 0 < tol < 1e-12), EMP_ERR_CUDA. */
int mp_model_radial_tables(void* model, double tol, int32_t* n_pieces);

/* The radial network p of `layer` on its own, in the model's current mode (network or
 * tables): for n lengths d [n], h2 [n][64] as its 3xTF32 split (h2_hi + h2_lo, the head's
 * operand), and, if g_h2 [n][64] is not NULL, dE_dd [n] = sum_j g_h2[j] dh2_j/dd.
 * Workspace >= 24 n + 256 bytes when g_h2 is given.  For inspecting the radial part
 * (e.g. the certificate of the tables); the energy and force calls do not need it. */
int mp_radial_hidden(const void* model, int32_t layer, int32_t pair, int64_t n, const float* d, float* h2_hi,
                     float* h2_lo, const float* g_h2, float* dE_dd, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes for mp_energy_forces at full speed: the layers between the first and the last
 * keep their per-edge mixing outputs y (n_edges x 16C floats each) from the forward for the
 * backward.  mp_workspace_bytes_min is the least mp_forward and mp_energy_forces accept: there
 * the backward recomputes y cohort by cohort (one more SO(2) product per edge and layer).
 * Any size from the minimum up runs; the path is chosen by the size passed, and both give the
 * same bits.  The sizes depend on the model's radial mode: with radial tables
 * (mp_model_radial_tables) the per-row hidden values take 768 bytes per edge more, so query
 * them after the tables are built (a workspace sized before them may be rejected with
 * EMP_ERR_WORKSPACE). */
size_t mp_workspace_bytes(const void* model, int64_t n_edges, int32_t n_atoms);
size_t mp_workspace_bytes_min(const void* model, int64_t n_edges, int32_t n_atoms);

/* One interaction layer (forward only): agg_out[i] = (1/avg_degree) * sum over
 * edges e with recv(e) = i of D(R_e)^T SO2_layer(R_e(d) (.) D(R_e) x_in[send(e)]).
 * species [N] int32 selects the radial network when pair_radial is set. */
int mp_forward(const void* model, const emp_graph* g, int32_t layer, const int32_t* species,
               const float* x_in, float* agg_out, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Energy and forces: energy (double[1]) = sum_i e_i, forces [N][3] = -dE/dx,
 * virial [9] = -sum_e r_e (x) dE/dr_e (row-major) or NULL, atom_energy [N] or NULL. */
int mp_energy_forces(const void* model, const emp_graph* g, const int32_t* species,
                     double* energy, float* forces, float* virial, float* atom_energy,
                     void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ multi-GPU: receiver ranges
 * Sum of a float buffer over all ranks, in place, ordered on `stream` (e.g. an NCCL
 * all-reduce); returns 0 on success.  Provided by the caller. */
typedef int (*emp_allreduce_fn)(float* buf, size_t n, cudaStream_t stream, void* ctx);

/* One rank's part of the energy + force step when the receivers are split into contiguous
 * ranges over ranks (one process per GPU): this rank computes the edges of receivers
 * [atom_begin, atom_end) of the whole graph g (every rank holds g and all node features).
 * After each layer's receiver sums, the sums are added over the ranks (allreduce; each
 * receiver's row comes from exactly one rank, so the sum is exact); in the backward, each
 * layer's gradient with respect to the layer's input is added over the ranks (the
 * residual part counted on rank 0 only), and at the end the per-edge gradients, so that
 * every rank returns the whole energy, forces, virial and atom energies.  The ranges must
 * cover the atoms, each once, over the ranks; any split is valid (balanced by edge count
 * for speed).  Workspace: mp_sharded_workspace_bytes(model, local edges, all edges, N) (y kept,
 * as for mp_workspace_bytes; down to (layers - 2) x local edges x 16C x 4 bytes less runs with y
 * recomputed).
 * Reads the range's edge offsets back to the host (synchronises once).  Not for CUDA-graph
 * capture unless allreduce is capturable. */
size_t mp_sharded_workspace_bytes(const void* model, int64_t n_edges_local, int64_t n_edges, int32_t n_atoms);
int mp_energy_forces_sharded(const void* model, const emp_graph* g, int32_t atom_begin, int32_t atom_end, int32_t rank,
                             const int32_t* species, double* energy, float* forces, float* virial, float* atom_energy,
                             emp_allreduce_fn allreduce, void* ctx, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Weight gradients of the energy (the training path, which the page "first-order SO(2)
 * input-gradient path" leaves on its old code path: "Implementation and scope"): energy,
 * forces, and grad [mp_weight_count] = dE/dW for every weight, in the blob order of
 * mp_weight_count (embedding, per layer the radial networks and the SO(2) blocks W0, Wr_m,
 * Wi_m, then the readout).  Sums over edges and nodes run in FP32 in a fixed order, so the
 * result is reproducible.  The radial hidden layers are the network's even when the model
 * has radial tables (their weights get gradients).  Gradients of force terms (mixed second
 * derivatives) are not computed.  Workspace: mp_weight_grad_workspace_bytes (larger than
 * mp_workspace_bytes: per-row radial values, block sums and reduction partials; like it, with y
 * kept, and down to (layers - 2) x edges x 16C x 4 bytes less with y recomputed). */
size_t mp_weight_grad_workspace_bytes(const void* model, int64_t n_edges, int32_t n_atoms);
int mp_energy_weight_grad(const void* model, const emp_graph* g, const int32_t* species, double* energy,
                          float* forces, float* grad, void* ws, size_t ws_bytes, cudaStream_t stream);

/* The per-m SO(2) channel mixing of a batch of edge-frame rows on its own
 * (page "first-order SO(2) input-gradient path": the mixing GEMMs, strict
 * FP32 -- here 3xTF32 on the tensor cores).  X, Y [M][16C] in the m-major
 * column layout [m=0 (l=0..3) | +1 (l=1..3) | -1 | +2 | -2 | +3 | -3], each
 * entry C channels.  transpose = 0: Y_b = X_b B_b^T (forward, y+ = Wr x+ - Wi x-,
 * y- = Wi x+ + Wr x-, y0 = W0 x0); transpose = 1: the adjoint map.
 * Workspace >= 2 * M * 16 * C floats (the TF32 split of X) + 256 bytes. */
int mp_so2_mix(const void* model, int32_t layer, int32_t transpose, int64_t M, const float* X, float* Y,
               void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------ radial chain
 * Page "deepmd-kit PR #6108: radial head fold", section "What": basis x
 * (E,4,32) -> per-degree up-projection U_l (32 -> 64) -> (E,256) @ M (256,25).
 * The chain object folds W_eff = vstack_l(U_l M_l) (128 x 25) once. */
int mp_chain_create(const float* U /*(host) [4][32][64] (in,out)*/,
                    const float* M /*(host) [256][25] (in,out)*/, void** chain /*(host) out*/);
void mp_chain_destroy(void* chain);

/* kc [E][25] = x_flat @ W_eff; y0 [E][64] = x[:,0,:] @ U_0.  If g_x is not
 * NULL also g_x [E][4][32] = g_kc @ W_eff^T (+ g_y0 @ U_0^T into degree 0).
 * Products on the tensor cores in 3xTF32 (FP32 accuracy).  x, g_kc, g_y0
 * row-major; 0 <= E < 2^31 - 128.  x, kc, y0, g_kc, g_y0 and g_x 16-byte
 * aligned (EMP_ERR_ARG otherwise: x and g_y0 are read by TMA, g_kc by bulk
 * copies, the outputs stored as float4). */
int mp_radial_chain(const void* chain, int64_t E, const float* x, float* kc, float* y0,
                    const float* g_kc, const float* g_y0, float* g_x, cudaStream_t stream);

/* ------------------------------------------------------------ timing
 * Every kernel launch of the library is counted.  With profiling enabled, a
 * pair of CUDA events is recorded on the launching stream around each launch,
 * grouped by kernel family ("so2_tc", "rotate_in", "rotate_back_scatter",
 * "bwd_prep", "bwd_edge", "sender_scatter", "radial_fwd", "radial_bwd",
 * "geometry", "nl", ...).  Host-side bookkeeping only; kernels are unchanged. */
int emp_profile_enable(int enable);                    /* also clears recorded events */
/* Device milliseconds and launch count of one family ("*" = all) recorded since
 * the last emp_profile_enable; synchronises on the recorded events. */
int emp_profile_read(const char* name, double* total_ms, int64_t* launches);
/* Comma-separated names of the families recorded so far, into buf[n]. */
int emp_profile_names(char* buf, size_t n);
int64_t emp_launch_count(void);                        /* kernels launched since the library was loaded */

/* ------------------------------------------------------------ status */
const char* emp_status_string(int status);
/* Reads and clears the device error word of the current device (synchronises). */
int emp_last_device_error(void);

/* ------------------------------------------------------------ tensor-pipe rate
 * Measures the TF32 rate of the tensor cores in the form the SO(2) products use
 * (tcgen05.mma.cta_group::2.kind::tf32, M = 256, N = 256, K = 8, operands resident in
 * shared memory): one CTA pair per two SMs issues `iters` rounds of twelve products, timed
 * with CUDA events on `stream` (synchronises).  tflops (host, out): TF32 flops per
 * second / 1e12, counting every product; a 3xTF32 product does three of them. */
int emp_tf32_mma_rate(int32_t iters, cudaStream_t stream, double* tflops);

/* ------------------------------------------------------------ bounded waits
 * Every mbarrier wait of the library's kernels gives up after a bound (clock64
 * cycles of the waiting SM), records EMP_ERR_TIMEOUT in the device error word,
 * stops issuing work, waits (bounded) for its own copies in flight and returns.
 * Sets the bound for the current device; cycles <= 0 restores the default
 * (4e9 cycles, about 2 s).  Synchronous with respect to the host. */
int emp_set_wait_limit(int64_t cycles);
/* Launches one bounded wait on an mbarrier that nothing arrives on: it runs out
 * after the bound in force, and emp_last_device_error() then reports
 * EMP_ERR_TIMEOUT.  For checking the failure path without a fault. */
int emp_wait_selftest(cudaStream_t stream);
/* The library rounds to TF32 (the 3xTF32 split: round to nearest, ties away from zero, at the
 * 10th mantissa bit) with integer operations on the bits.  This runs that rounding and the
 * conversion instruction cvt.rna.tf32.f32 on every 32-bit pattern that is not a NaN and stores
 * in *mismatches how many differ (0 expected).  Allocates 8 bytes of device memory; synchronous.
 * Errors: EMP_ERR_ARG (null), EMP_ERR_UNSUPPORTED (not sm_100), EMP_ERR_CUDA. */
int emp_tf32_split_selftest(uint64_t* mismatches);

#ifdef __cplusplus
}
#endif
#endif /* EMP_H */
