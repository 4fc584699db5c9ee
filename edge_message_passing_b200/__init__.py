"""Python binding of the B200 equivariant edge message-passing library (libemp.so).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  There is
no CPU fallback: importing works without a GPU, but every compute call needs
the compiled library and a CUDA device, and raises otherwise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libemp.so")

# exported symbols (kept in step with include/emp.h)
SYMBOLS = (
    "nl_workspace_bytes", "nl_build", "nl_build_noalloc", "mp_weight_count", "mp_model_create", "mp_model_destroy",
    "mp_workspace_bytes", "mp_workspace_bytes_min", "mp_forward", "mp_energy_forces", "mp_so2_mix", "mp_chain_create",
    "mp_chain_destroy", "mp_radial_chain", "emp_status_string", "emp_last_device_error",
    "emp_profile_enable", "emp_profile_read", "emp_profile_names", "emp_launch_count",
    "emp_set_wait_limit", "emp_wait_selftest", "emp_tf32_split_selftest", "emp_tf32_mma_rate", "mp_model_radial_tables", "mp_radial_hidden",
    "mp_weight_grad_workspace_bytes", "mp_energy_weight_grad", "nl_refresh",
    "mp_sharded_workspace_bytes", "mp_energy_forces_sharded",
)

# int (*)(float* buf, size_t n, cudaStream_t stream, void* ctx): the sum over ranks, in place
ALLREDUCE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p)


class EmpError(RuntimeError):
    pass


class NlParams(ctypes.Structure):
    _fields_ = [("n_atoms", ctypes.c_int32), ("box", ctypes.c_double * 3), ("cutoff", ctypes.c_double),
                ("capacity", ctypes.c_int64)]


class GraphC(ctypes.Structure):
    _fields_ = [("recv", ctypes.c_void_p), ("send", ctypes.c_void_p), ("mirror", ctypes.c_void_p),
                ("recv_off", ctypes.c_void_p), ("shift", ctypes.c_void_p), ("vec", ctypes.c_void_p),
                ("n_edges", ctypes.c_int64), ("n_atoms", ctypes.c_int32)]


class SpecC(ctypes.Structure):
    _fields_ = [("C", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("n_species", ctypes.c_int32),
                ("n_basis", ctypes.c_int32), ("radial_hidden", ctypes.c_int32),
                ("readout_hidden", ctypes.c_int32), ("gated", ctypes.c_int32),
                ("pair_radial", ctypes.c_int32), ("cohort_edges", ctypes.c_int32),
                ("cutoff", ctypes.c_float), ("env_p", ctypes.c_int32), ("avg_degree", ctypes.c_float)]


_lib_handle = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise EmpError(f"{LIB_PATH} is missing: build it with `python -m edge_message_passing_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.nl_workspace_bytes.restype = sz
        L.nl_workspace_bytes.argtypes = [i32]
        L.nl_build.restype = ctypes.c_int
        L.nl_build.argtypes = [ctypes.POINTER(NlParams), vp, ctypes.POINTER(GraphC), ctypes.POINTER(i64), vp, sz, vp]
        L.nl_build_noalloc.restype = ctypes.c_int
        L.nl_build_noalloc.argtypes = [ctypes.POINTER(NlParams), vp, ctypes.POINTER(GraphC), ctypes.POINTER(i64), vp]
        L.mp_sharded_workspace_bytes.restype = sz
        L.mp_sharded_workspace_bytes.argtypes = [vp, i64, i64, i32]
        L.mp_energy_forces_sharded.restype = ctypes.c_int
        L.mp_energy_forces_sharded.argtypes = [vp, ctypes.POINTER(GraphC), i32, i32, i32, vp, vp, vp, vp, vp,
                                               ALLREDUCE_FN, vp, vp, sz, vp]
        L.nl_refresh.restype = ctypes.c_int
        L.nl_refresh.argtypes = [ctypes.POINTER(NlParams), vp, vp, ctypes.c_double, ctypes.POINTER(GraphC),
                                 ctypes.POINTER(i32), vp, sz, vp]
        L.mp_weight_count.restype = sz
        L.mp_weight_count.argtypes = [ctypes.POINTER(SpecC)]
        L.mp_model_create.restype = ctypes.c_int
        L.mp_model_create.argtypes = [ctypes.POINTER(SpecC), vp, sz, ctypes.POINTER(vp)]
        L.mp_model_destroy.restype = None
        L.mp_model_destroy.argtypes = [vp]
        L.mp_workspace_bytes.restype = sz
        L.mp_workspace_bytes.argtypes = [vp, i64, i32]
        L.mp_workspace_bytes_min.restype = sz
        L.mp_workspace_bytes_min.argtypes = [vp, i64, i32]
        L.mp_forward.restype = ctypes.c_int
        L.mp_forward.argtypes = [vp, ctypes.POINTER(GraphC), i32, vp, vp, vp, vp, sz, vp]
        L.mp_energy_forces.restype = ctypes.c_int
        L.mp_energy_forces.argtypes = [vp, ctypes.POINTER(GraphC), vp, vp, vp, vp, vp, vp, sz, vp]
        L.mp_so2_mix.restype = ctypes.c_int
        L.mp_so2_mix.argtypes = [vp, i32, i32, i64, vp, vp, vp, sz, vp]
        L.mp_chain_create.restype = ctypes.c_int
        L.mp_chain_create.argtypes = [vp, vp, ctypes.POINTER(vp)]
        L.mp_chain_destroy.restype = None
        L.mp_chain_destroy.argtypes = [vp]
        L.mp_radial_chain.restype = ctypes.c_int
        L.mp_radial_chain.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, vp]
        L.emp_status_string.restype = ctypes.c_char_p
        L.emp_status_string.argtypes = [ctypes.c_int]
        L.emp_last_device_error.restype = ctypes.c_int
        L.emp_last_device_error.argtypes = []
        L.emp_profile_enable.restype = ctypes.c_int
        L.emp_profile_enable.argtypes = [ctypes.c_int]
        L.emp_profile_read.restype = ctypes.c_int
        L.emp_profile_read.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)]
        L.emp_profile_names.restype = ctypes.c_int
        L.emp_profile_names.argtypes = [ctypes.c_char_p, sz]
        L.emp_launch_count.restype = i64
        L.emp_launch_count.argtypes = []
        L.emp_set_wait_limit.restype = ctypes.c_int
        L.emp_set_wait_limit.argtypes = [i64]
        L.emp_wait_selftest.restype = ctypes.c_int
        L.emp_wait_selftest.argtypes = [vp]
        L.emp_tf32_split_selftest.restype = ctypes.c_int
        L.emp_tf32_split_selftest.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
        L.mp_weight_grad_workspace_bytes.restype = sz
        L.mp_weight_grad_workspace_bytes.argtypes = [vp, i64, i32]
        L.mp_energy_weight_grad.restype = ctypes.c_int
        L.mp_energy_weight_grad.argtypes = [vp, ctypes.POINTER(GraphC), vp, vp, vp, vp, vp, sz, vp]
        L.mp_model_radial_tables.restype = ctypes.c_int
        L.mp_model_radial_tables.argtypes = [vp, ctypes.c_double, ctypes.POINTER(i32)]
        L.mp_radial_hidden.restype = ctypes.c_int
        L.mp_radial_hidden.argtypes = [vp, i32, i32, i64, vp, vp, vp, vp, vp, vp, sz, vp]
        L.emp_tf32_mma_rate.restype = ctypes.c_int
        L.emp_tf32_mma_rate.argtypes = [i32, vp, ctypes.POINTER(ctypes.c_double)]
        _lib_handle = L
    return _lib_handle


def _check(status: int, what: str) -> None:
    if status != 0:
        raise EmpError(f"{what}: {lib().emp_status_string(status).decode()} ({status})")


def _torch():
    import torch
    if not torch.cuda.is_available():
        raise EmpError("a CUDA device is required")
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream():
    return _torch().cuda.current_stream().cuda_stream


def last_device_error() -> int:
    """Read and clear the device error word (0 = none)."""
    return lib().emp_last_device_error()


def set_wait_limit(cycles: int = 0) -> None:
    """Bound (clock64 cycles) of every device-side wait; 0 restores the default (~2 s)."""
    _check(lib().emp_set_wait_limit(int(cycles)), "emp_set_wait_limit")


def wait_selftest() -> int:
    """One bounded wait that nothing satisfies; returns the device error it records."""
    _check(lib().emp_wait_selftest(_stream()), "emp_wait_selftest")
    return last_device_error()


def tf32_split_selftest() -> int:
    """Patterns (of all non-NaN 32-bit ones) where the library's TF32 rounding differs from
    cvt.rna.tf32.f32 (0 expected)."""
    n = ctypes.c_uint64(0)
    _check(lib().emp_tf32_split_selftest(ctypes.byref(n)), "emp_tf32_split_selftest")
    return int(n.value)


def tf32_mma_rate(iters: int = 20000) -> float:
    """TF32 TFLOP/s of the tensor cores in the SO(2) products' form (operands resident in
    shared memory); a 3xTF32 product costs three."""
    v = ctypes.c_double(0.0)
    _check(lib().emp_tf32_mma_rate(int(iters), _stream(), ctypes.byref(v)), "emp_tf32_mma_rate")
    return v.value


def profile_enable(on: bool = True) -> None:
    """Start (or stop) per-kernel CUDA-event timing; clears what was recorded."""
    _check(lib().emp_profile_enable(int(on)), "emp_profile_enable")


def profile_read(name: str = "*"):
    """(device milliseconds, launches) of one kernel family since profile_enable."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int64(0)
    _check(lib().emp_profile_read(name.encode(), ctypes.byref(ms), ctypes.byref(n)), "emp_profile_read")
    return ms.value, n.value


def profile_names() -> list:
    buf = ctypes.create_string_buffer(4096)
    _check(lib().emp_profile_names(buf, 4096), "emp_profile_names")
    return [x for x in buf.value.decode().split(",") if x]


def launch_count() -> int:
    return int(lib().emp_launch_count())


_ws_cache: Dict[int, object] = {}


def _workspace(nbytes: int):
    """A device scratch buffer of at least nbytes (cached per device)."""
    torch = _torch()
    dev = torch.cuda.current_device()
    buf = _ws_cache.get(dev)
    if buf is None or buf.numel() < nbytes:
        _ws_cache.pop(dev, None)
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
        _ws_cache[dev] = buf
    return buf


# ------------------------------------------------------------------ neighbour list
@dataclasses.dataclass
class Graph:
    recv: object
    send: object
    mirror: object
    recv_off: object
    shift: object
    vec: object
    n_edges: int
    n_atoms: int

    def c(self) -> GraphC:
        return GraphC(_ptr(self.recv), _ptr(self.send), _ptr(self.mirror), _ptr(self.recv_off),
                      _ptr(self.shift), _ptr(self.vec), self.n_edges, self.n_atoms)


def nl_build(pos, box: Sequence[float], cutoff: float, capacity: Optional[int] = None,
             reuse: Optional["Graph"] = None) -> Graph:
    """Neighbour list of device positions pos [N,3] float64 (see include/emp.h).

    reuse: a Graph from an earlier call whose buffers are written again when they
    are large enough (same atom count), instead of allocating new ones."""
    torch = _torch()
    if pos.dtype != torch.float64 or pos.dim() != 2 or pos.shape[1] != 3 or not pos.is_cuda:
        raise EmpError("pos must be a CUDA float64 tensor [N,3]")
    pos = pos.contiguous()
    N = pos.shape[0]
    L = lib()
    ws = _workspace(L.nl_workspace_bytes(N))
    cap = capacity if capacity is not None else max(256, 200 * N)
    bufs = None
    if reuse is not None and reuse.n_atoms == N and getattr(reuse, "_full", None) is not None:
        bufs = reuse._full
        cap = bufs[0].shape[0]
    for _ in range(2):
        if bufs is None or bufs[0].shape[0] < cap:
            bufs = (*(torch.empty(cap, dtype=torch.int32, device="cuda") for _ in range(3)),
                    torch.empty(N + 1, dtype=torch.int32, device="cuda"),
                    torch.empty((cap, 3), dtype=torch.int32, device="cuda"),
                    torch.empty((cap, 3), dtype=torch.float32, device="cuda"))
        g = Graph(*bufs, 0, N)
        p = NlParams(N, (ctypes.c_double * 3)(*[float(b) for b in box]), float(cutoff), cap)
        gc = g.c()
        ne = ctypes.c_int64(0)
        st = L.nl_build(ctypes.byref(p), _ptr(pos), ctypes.byref(gc), ctypes.byref(ne), _ptr(ws), ws.numel(),
                        _stream())
        if st == -2 and ne.value > cap:           # capacity: grow once to the reported size
            cap = int(ne.value)
            bufs = None
            continue
        _check(st, "nl_build")
        E = int(ne.value)
        out = Graph(bufs[0][:E], bufs[1][:E], bufs[2][:E], bufs[3], bufs[4][:E], bufs[5][:E], E, N)
        out._full = bufs
        return out
    raise EmpError("nl_build: capacity retry failed")


def nl_refresh(graph: Graph, pos, pos_ref, box: Sequence[float], skin: float) -> bool:
    """Edge vectors of `graph` (built with cutoff + skin at pos_ref) at positions pos; True when
    some atom moved more than skin / 2 from pos_ref (the graph must then be built again)."""
    torch = _torch()
    pos = pos.contiguous()
    ws = _workspace(256)
    p = NlParams(graph.n_atoms, (ctypes.c_double * 3)(*[float(b) for b in box]), 0.0, graph.n_edges)
    gc = graph.c()
    flag = ctypes.c_int32(0)
    _check(lib().nl_refresh(ctypes.byref(p), _ptr(pos), _ptr(pos_ref), float(skin), ctypes.byref(gc),
                            ctypes.byref(flag), _ptr(ws), ws.numel(), _stream()), "nl_refresh")
    return bool(flag.value)


class NeighbourCache:
    """Neighbour list for an MD loop: built with cutoff + skin and reused, with its edge vectors
    refreshed at every call, until some atom has moved more than skin / 2 since the build."""

    def __init__(self, box: Sequence[float], cutoff: float, skin: float):
        self.box, self.cutoff, self.skin = list(box), float(cutoff), float(skin)
        self.graph, self.pos_ref, self.builds = None, None, 0

    def update(self, pos) -> Graph:
        if self.graph is not None and not nl_refresh(self.graph, pos, self.pos_ref, self.box, self.skin):
            return self.graph
        self.graph = nl_build(pos, self.box, self.cutoff + self.skin, reuse=self.graph)
        self.pos_ref = pos.clone()
        self.builds += 1
        return self.graph


# ------------------------------------------------------------------ model
def weight_order(spec) -> list:
    """Weight names in the blob order documented in include/emp.h."""
    names = ["emb"]
    n_pairs = spec.n_species * (spec.n_species + 1) // 2 if spec.pair_radial else 1
    for t in range(spec.n_layers):
        for p in range(n_pairs):
            names += [f"rad{t}_{p}_W1", f"rad{t}_{p}_W2", f"rad{t}_{p}_W3"]
        names.append(f"so2_{t}_W0")
        for m in (1, 2, 3):
            names += [f"so2_{t}_Wr{m}", f"so2_{t}_Wi{m}"]
    return names + ["ro_W", "ro_w"]


def spec_c(spec) -> SpecC:
    return SpecC(spec.C, spec.n_layers, spec.n_species, spec.n_basis, spec.radial_hidden,
                 spec.readout_hidden if spec.readout_hidden > 0 else spec.C, int(spec.gated),
                 int(spec.pair_radial), spec.cohort_edges, float(spec.cutoff), spec.env_p,
                 float(spec.avg_degree))


class Model:
    """Device model: weights copied, SO(2) blocks stacked and split for 3xTF32."""

    def __init__(self, spec, weights: Dict[str, np.ndarray]):
        _torch()
        self.spec = spec
        sc = spec_c(spec)
        blob = np.concatenate([np.ascontiguousarray(weights[k], dtype=np.float32).ravel()
                               for k in weight_order(spec)])
        self.shapes = [(k, tuple(np.shape(weights[k]))) for k in weight_order(spec)]
        n = lib().mp_weight_count(ctypes.byref(sc))
        if n != blob.size:
            raise EmpError(f"weight blob has {blob.size} floats, the library expects {n}")
        h = ctypes.c_void_p()
        _check(lib().mp_model_create(ctypes.byref(sc), blob.ctypes.data, blob.size, ctypes.byref(h)),
               "mp_model_create")
        self.handle = h.value

    def workspace_bytes(self, n_edges: int, n_atoms: int) -> int:
        return lib().mp_workspace_bytes(self.handle, n_edges, n_atoms)

    def workspace_bytes_min(self, n_edges: int, n_atoms: int) -> int:
        return lib().mp_workspace_bytes_min(self.handle, n_edges, n_atoms)

    def radial_tables(self, tol: float = 1e-7) -> int:
        """Switch the radial hidden layers to certified Chebyshev tables (tol > 0; returns
        the number of pieces) or back to the network (tol <= 0)."""
        n = ctypes.c_int32(0)
        _check(lib().mp_model_radial_tables(self.handle, float(tol), ctypes.byref(n)), "mp_model_radial_tables")
        return n.value

    def __del__(self):
        if getattr(self, "handle", None) and _lib_handle is not None:
            _lib_handle.mp_model_destroy(self.handle)
            self.handle = None


def mp_forward(model: Model, graph: Graph, layer: int, species, x):
    """One interaction layer: agg [N,16,C] for node features x [N,16,C] (float32, CUDA)."""
    torch = _torch()
    x = x.contiguous()
    agg = torch.empty_like(x)
    ws = _workspace(model.workspace_bytes_min(graph.n_edges, graph.n_atoms))
    gc = graph.c()
    _check(lib().mp_forward(model.handle, ctypes.byref(gc), layer, _ptr(species), _ptr(x), _ptr(agg), _ptr(ws),
                            ws.numel(), _stream()), "mp_forward")
    return agg


def mp_energy_forces(model: Model, graph: Graph, species, virial: bool = False, atom_energy: bool = False,
                     compact: bool = False):
    """(energy [1] float64, forces [N,3], virial [3,3] or None, atom energies [N] or None).
    compact: run in the smallest workspace (the backward recomputes the per-edge mixing outputs
    instead of keeping them from the forward); the results are the same bits."""
    torch = _torch()
    N = graph.n_atoms
    energy = torch.empty(1, dtype=torch.float64, device="cuda")
    forces = torch.empty((N, 3), dtype=torch.float32, device="cuda")
    vir = torch.empty((3, 3), dtype=torch.float32, device="cuda") if virial else None
    ea = torch.empty(N, dtype=torch.float32, device="cuda") if atom_energy else None
    nbytes = (model.workspace_bytes_min if compact else model.workspace_bytes)(graph.n_edges, N)
    ws = _workspace(nbytes)
    gc = graph.c()
    _check(lib().mp_energy_forces(model.handle, ctypes.byref(gc), _ptr(species), _ptr(energy), _ptr(forces),
                                  _ptr(vir), _ptr(ea), _ptr(ws), nbytes, _stream()), "mp_energy_forces")
    return energy, forces, vir, ea


def mp_energy_weight_grad(model: Model, graph: Graph, species):
    """(energy [1] float64, forces [N,3], {weight name: dE/dW} as CUDA float32 tensors shaped like
    the weights) -- the weight gradient of the energy (the training path)."""
    torch = _torch()
    N = graph.n_atoms
    energy = torch.empty(1, dtype=torch.float64, device="cuda")
    forces = torch.empty((N, 3), dtype=torch.float32, device="cuda")
    sc = spec_c(model.spec)
    n = lib().mp_weight_count(ctypes.byref(sc))
    grad = torch.empty(n, dtype=torch.float32, device="cuda")
    ws = _workspace(lib().mp_weight_grad_workspace_bytes(model.handle, graph.n_edges, N))
    gc = graph.c()
    _check(lib().mp_energy_weight_grad(model.handle, ctypes.byref(gc), _ptr(species), _ptr(energy), _ptr(forces),
                                       _ptr(grad), _ptr(ws), ws.numel(), _stream()), "mp_energy_weight_grad")
    out, o = {}, 0
    for name, shape in model.shapes:
        k = int(np.prod(shape))
        out[name] = grad[o:o + k].view(*shape)
        o += k
    return energy, forces, out


def receiver_ranges(recv_off, world: int):
    """Contiguous receiver ranges [(a, b)] for `world` ranks, cut where the running edge count
    crosses r E / world (balanced by edges, each atom in exactly one range)."""
    ro = np.asarray(recv_off, dtype=np.int64)
    N, E = ro.shape[0] - 1, int(ro[-1])
    cuts = [0] + [int(np.searchsorted(ro, r * E / world, side="left")) for r in range(1, world)] + [N]
    cuts = np.minimum(np.maximum.accumulate(np.asarray(cuts)), N)
    return [(int(cuts[r]), int(cuts[r + 1])) for r in range(world)]


def mp_energy_forces_sharded(model: Model, graph: Graph, species, rank: int, world: int, group=None,
                             virial: bool = False):
    """This rank's part of the energy + force step over receiver ranges (one process per GPU,
    torch.distributed initialised): returns the whole (energy, forces, virial or None) on every
    rank.  The sums over ranks go through torch.distributed.all_reduce (NCCL on the GPU; with the
    gloo backend through host copies)."""
    import torch.distributed as dist
    torch = _torch()
    N = graph.n_atoms
    a, b = receiver_ranges(graph.recv_off.cpu().numpy(), world)[rank]
    ro = graph.recv_off.cpu().numpy()
    El = int(ro[b] - ro[a])
    ws = _workspace(lib().mp_sharded_workspace_bytes(model.handle, El, graph.n_edges, N))
    gloo = dist.get_backend(group) == "gloo"
    base = ws.data_ptr()

    def allreduce(buf, n, stream, ctx):
        try:
            t = ws[buf - base: buf - base + 4 * n].view(torch.float32)
            if gloo:
                h = t.cpu()
                dist.all_reduce(h, group=group)
                t.copy_(h)
            else:
                dist.all_reduce(t, group=group)
            return 0
        except Exception:                     # no exception crosses the C ABI: report a failure
            return 1

    fn = ALLREDUCE_FN(allreduce)
    energy = torch.empty(1, dtype=torch.float64, device="cuda")
    forces = torch.empty((N, 3), dtype=torch.float32, device="cuda")
    vir = torch.empty((3, 3), dtype=torch.float32, device="cuda") if virial else None
    gc = graph.c()
    _check(lib().mp_energy_forces_sharded(model.handle, ctypes.byref(gc), a, b, rank, _ptr(species), _ptr(energy),
                                          _ptr(forces), _ptr(vir), None, fn, None, _ptr(ws), ws.numel(), _stream()),
           "mp_energy_forces_sharded")
    return energy, forces, vir


class EnergyForcesGraph:
    """mp_energy_forces of one neighbour graph and species array, captured once as a
    CUDA graph and replayed.  The replay runs the library's own kernels with the
    pointers captured here: the outputs (energy, forces, virial, atom_energy) are
    this object's tensors, overwritten by every replay, and graph, species and the
    workspace are kept alive by the object.  The positions must not change between
    replays without a new capture (the graph's edge vectors are inputs).  compact: the smallest
    workspace (the backward recomputes the per-edge mixing outputs; the same bits)."""

    def __init__(self, model: Model, graph: Graph, species, virial: bool = False, atom_energy: bool = False,
                 compact: bool = False):
        torch = _torch()
        N = graph.n_atoms
        self.model, self.graph, self.species = model, graph, species
        self.energy = torch.empty(1, dtype=torch.float64, device="cuda")
        self.forces = torch.empty((N, 3), dtype=torch.float32, device="cuda")
        self.virial = torch.empty((3, 3), dtype=torch.float32, device="cuda") if virial else None
        self.atom_energy = torch.empty(N, dtype=torch.float32, device="cuda") if atom_energy else None
        nbytes = (model.workspace_bytes_min if compact else model.workspace_bytes)(graph.n_edges, N)
        self.ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
        self._gc = graph.c()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self._call()                      # first call outside the capture (one-time set-up)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.cuda_graph = torch.cuda.CUDAGraph()
        n0 = launch_count()
        with torch.cuda.graph(self.cuda_graph):
            self._call()
        self.launches = launch_count() - n0   # library kernels per replay

    def _call(self):
        _check(lib().mp_energy_forces(self.model.handle, ctypes.byref(self._gc), _ptr(self.species),
                                      _ptr(self.energy), _ptr(self.forces), _ptr(self.virial),
                                      _ptr(self.atom_energy), _ptr(self.ws), self.ws.numel(), _stream()),
               "mp_energy_forces")

    def replay(self):
        self.cuda_graph.replay()
        return self.energy, self.forces, self.virial, self.atom_energy


def mp_radial_hidden(model: Model, layer: int, pair: int, d, g_h2=None):
    """Radial network `pair` of `layer` at lengths d [n] (CUDA float32), in the model's current
    mode: (h2 hi [n,64], h2 lo [n,64], dE/dd [n] for dE/dh2 = g_h2, or None)."""
    torch = _torch()
    d = d.contiguous()
    n = d.shape[0]
    hi = torch.empty((n, 64), dtype=torch.float32, device="cuda")
    lo = torch.empty_like(hi)
    dEdd = torch.empty(n, dtype=torch.float32, device="cuda") if g_h2 is not None else None
    g = None if g_h2 is None else g_h2.contiguous()
    ws = _workspace(24 * n + 256)
    _check(lib().mp_radial_hidden(model.handle, layer, pair, n, _ptr(d), _ptr(hi), _ptr(lo), _ptr(g), _ptr(dEdd),
                                  _ptr(ws), ws.numel(), _stream()), "mp_radial_hidden")
    return hi, lo, dEdd


def mp_so2_mix(model: Model, layer: int, X, transpose: bool = False):
    """The per-m SO(2) block products of X [M,16C] (m-major column layout)."""
    torch = _torch()
    X = X.contiguous()
    Y = torch.empty_like(X)
    ws = _workspace(2 * X.numel() * 4 + 256)
    _check(lib().mp_so2_mix(model.handle, layer, int(transpose), X.shape[0], _ptr(X), _ptr(Y), _ptr(ws),
                            ws.numel(), _stream()), "mp_so2_mix")
    return Y


# ------------------------------------------------------------------ radial chain
class Chain:
    """Folded radial projection chain (W_eff formed once on the device)."""

    def __init__(self, U: np.ndarray, M: np.ndarray):
        _torch()
        U = np.ascontiguousarray(U, dtype=np.float32)
        M = np.ascontiguousarray(M, dtype=np.float32)
        if U.shape != (4, 32, 64) or M.shape != (256, 25):
            raise EmpError("U must be [4,32,64] and M [256,25]")
        h = ctypes.c_void_p()
        _check(lib().mp_chain_create(U.ctypes.data, M.ctypes.data, ctypes.byref(h)), "mp_chain_create")
        self.handle = h.value

    def __del__(self):
        if getattr(self, "handle", None) and _lib_handle is not None:
            _lib_handle.mp_chain_destroy(self.handle)
            self.handle = None


def mp_radial_chain(chain: Chain, x, g_kc=None, g_y0=None, out=None):
    """(kc [E,25], y0 [E,64], g_x [E,4,32] or None) for x [E,4,32] float32 CUDA."""
    torch = _torch()
    x = x.contiguous()
    E = x.shape[0]
    if out is None:
        kc = torch.empty((E, 25), dtype=torch.float32, device="cuda")
        y0 = torch.empty((E, 64), dtype=torch.float32, device="cuda")
        gx = torch.empty_like(x) if g_kc is not None else None
    else:
        kc, y0, gx = out
    _check(lib().mp_radial_chain(chain.handle, E, _ptr(x), _ptr(kc), _ptr(y0), _ptr(g_kc), _ptr(g_y0), _ptr(gx),
                                 _stream()), "mp_radial_chain")
    return kc, y0, gx
