"""ctypes binding of the C ABI in include/afd_ffn.h (argument marshalling only).

Every step of the layer runs in the CUDA library; this module never computes any part of
it. PyTorch supplies device memory and streams. If the library is missing the import of
`lib()` raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_uint8, c_void_p
from typing import Optional, Sequence

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libafd_ffn.so")

AFD_OK = 0
STATUS_NAMES = {0: "AFD_OK", 1: "AFD_ERR_INVALID_ARGUMENT", 2: "AFD_ERR_UNSUPPORTED",
                3: "AFD_ERR_OUT_OF_MEMORY", 4: "AFD_ERR_CUDA", 5: "AFD_ERR_BAD_ROUTING",
                6: "AFD_ERR_TIMEOUT"}
STATUS_BAD_ROUTING, STATUS_TIMEOUT, STATUS_BAD_COUNT, STATUS_BAD_SCALE = 0x1, 0x2, 0x4, 0x8
KERNEL_NAMES = ["route_count", "route_scan", "route_scatter", "gather_rows", "gemm13_swiglu",
                "gemm2_combine", "combine_finalize"]


class Config(ctypes.Structure):
    _fields_ = [("hidden", c_int32), ("intermediate", c_int32), ("num_experts_global", c_int32),
                ("expert_begin", c_int32), ("num_local_experts", c_int32),
                ("has_shared_expert", c_int32), ("top_k", c_int32), ("num_slabs", c_int32),
                ("slab_capacity", c_int32)]


class Weights(ctypes.Structure):
    _fields_ = [("w13", c_void_p), ("w13_scale", c_void_p), ("w2", c_void_p), ("w2_scale", c_void_p)]


class SlabDesc(ctypes.Structure):
    _fields_ = [("x", c_void_p), ("x_scale", c_void_p), ("topk_ids", c_void_p),
                ("topk_weights", c_void_p), ("y", c_void_p)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_groups", c_int32), ("max_tokens", c_int32), ("max_rows", c_int32),
                ("num_sms", c_int32), ("workspace_bytes", c_int64)]


class BoundSlabs:
    """A slab set marshalled by FfnLayer.bind: the descriptor array and the counts pointer
    (the tensors are kept referenced)."""

    def __init__(self, descs, counts, keep):
        self.descs = descs
        self.counts = counts
        self._keep = keep


class AfdError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load libafd_ffn.so (built in-tree by build.py). Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run attention_ffn_disaggregated_b200/build.py)")
    L = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    sig = {
        "afd_ffn_check_config": (c_int32, [POINTER(Config)]),
        "afd_ffn_plan": (c_int32, [POINTER(Config), POINTER(Weights), POINTER(c_void_p)]),
        "afd_ffn_layer": (c_int32, [P, POINTER(SlabDesc), P, P]),
        "afd_ffn_destroy": (None, [P]),
        "afd_ffn_get_info": (c_int32, [P, POINTER(PlanInfo)]),
        "afd_ffn_get_status": (c_int32, [P, P, POINTER(c_int32)]),
        "afd_ffn_read_routing": (c_int32, [P, P, POINTER(c_int32), POINTER(c_int32), P, P, P, P, P, P]),
        "afd_ffn_read_intermediate": (c_int32, [P, P, P, P]),
        "afd_ffn_set_timing": (c_int32, [P, c_int32]),
        "afd_ffn_get_kernel_times": (c_int32, [P, POINTER(c_float)]),
        "afd_ffn_set_wait_limit": (c_int32, [P, c_int64]),
        "afd_ffn_inject_stall": (c_int32, [P, c_int32]),
        "afd_ffn_set_tiling": (c_int32, [P, c_int32]),
        "afd_ffn_get_tiling": (c_int32, [P, P, POINTER(c_int32)]),
        "afd_ffn_kernels_per_layer": (c_int32, [P]),
        "afd_ffn_set_combine_targets": (c_int32, [P, P]),
        "afd_combine_finalize": (c_int32, [POINTER(SlabDesc), c_int32, c_int32, c_int32, P, P, P]),
        "afd_ffn_route_noalloc": (c_int32, [POINTER(Config), POINTER(SlabDesc), P, P, P, P, P, P, P, P,
                                            P, P]),
        "afd_status_string": (c_char_p, [c_int32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def make_config(shape, num_slabs: int, slab_capacity: int) -> Config:
    return Config(shape.hidden, shape.intermediate, shape.num_experts_global, shape.expert_begin,
                  shape.num_local_experts, shape.has_shared_expert, shape.top_k, num_slabs,
                  slab_capacity)


def check_config(cfg: Config) -> int:
    return lib().afd_ffn_check_config(ctypes.byref(cfg))


def _ptr(t, name: str = "tensor") -> Optional[int]:
    """Device address of a CUDA tensor (None stays None). The kernels read these addresses
    as dense device arrays, so host or strided tensors are refused here rather than
    handed to the GPU."""
    if t is None:
        return None
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    h = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return h or None


class FfnLayer:
    """One FFN-pool expert layer on the current CUDA device.

    w13/w13_scale/w2/w2_scale: CUDA tensors in the layouts of include/afd_ffn.h (uint8 codes,
    float32 scales); they are kept referenced for the plan's lifetime.
    """

    def __init__(self, shape, num_slabs: int, slab_capacity: int, w13, w13_scale, w2, w2_scale):
        L = lib()
        self.shape = shape
        self.num_slabs = num_slabs
        self.slab_capacity = slab_capacity
        self._keep = (w13, w13_scale, w2, w2_scale)
        self.cfg = make_config(shape, num_slabs, slab_capacity)
        w = Weights(_ptr(w13, "w13"), _ptr(w13_scale, "w13_scale"), _ptr(w2, "w2"),
                    _ptr(w2_scale, "w2_scale"))
        h = c_void_p()
        rc = L.afd_ffn_plan(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(h))
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_plan")
        self.plan = h
        self.info = PlanInfo()
        L.afd_ffn_get_info(self.plan, ctypes.byref(self.info))

    def close(self):
        if getattr(self, "plan", None):
            lib().afd_ffn_destroy(self.plan)
            self.plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def bind(self, slabs: Sequence, counts) -> "BoundSlabs":
        """Marshal a slab set once (its device pointers, checked) for repeated calls: a
        serving loop whose receive buffers are fixed passes the result to __call__ instead
        of the slabs, so that a call costs one C call on the host."""
        if len(slabs) != self.num_slabs:
            raise ValueError("expected %d slabs" % self.num_slabs)
        descs = (SlabDesc * self.num_slabs)()
        for i, s in enumerate(slabs):
            descs[i] = SlabDesc(_ptr(s.x, "x"), _ptr(s.x_scale, "x_scale"), _ptr(s.topk_ids, "topk_ids"),
                                _ptr(s.topk_weights, "topk_weights"), _ptr(s.y, "y"))
        return BoundSlabs(descs, c_void_p(_ptr(counts, "counts")), (slabs, counts))

    def __call__(self, slabs, counts=None, stream=None) -> None:
        """slabs: a sequence of objects with .x .x_scale .topk_ids .topk_weights .y CUDA
        tensors and counts a device int32 tensor, or a BoundSlabs from bind() (counts None)."""
        b = slabs if isinstance(slabs, BoundSlabs) else self.bind(slabs, counts)
        rc = lib().afd_ffn_layer(self.plan, b.descs, b.counts, c_void_p(_stream_handle(stream)))
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_layer")

    def status(self, stream=None):
        word = c_int32(0)
        rc = lib().afd_ffn_get_status(self.plan, c_void_p(_stream_handle(stream)), ctypes.byref(word))
        return rc, word.value

    def routing(self, stream=None) -> dict:
        inf = self.info
        G, R, T = inf.num_groups, inf.max_rows, inf.max_tokens
        K = self.shape.top_k
        nt, nr = c_int32(0), c_int32(0)
        counts = np.zeros(G, np.int32)
        offsets = np.zeros(G + 1, np.int32)
        row_token = np.zeros(max(R, 1), np.int32)
        row_k = np.zeros(max(R, 1), np.int32)
        row_w = np.zeros(max(R, 1), np.float32)
        pos = np.zeros(max(T * K, 1), np.int32)
        rc = lib().afd_ffn_read_routing(
            self.plan, c_void_p(_stream_handle(stream)), ctypes.byref(nt), ctypes.byref(nr),
            counts.ctypes.data, offsets.ctypes.data, row_token.ctypes.data, row_k.ctypes.data,
            row_w.ctypes.data, pos.ctypes.data)
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_read_routing")
        r = nr.value
        return {"num_tokens": nt.value, "num_rows": r, "counts": counts, "offsets": offsets,
                "row_token": row_token[:r], "row_k": row_k[:r], "row_weight": row_w[:r],
                "pos": pos[:nt.value * K]}

    def intermediate(self, stream=None):
        R = self.info.max_rows
        I = self.shape.intermediate
        codes = np.zeros((max(R, 1), I), np.uint8)
        scales = np.zeros((max(R, 1), I // 128), np.float32)
        rc = lib().afd_ffn_read_intermediate(self.plan, c_void_p(_stream_handle(stream)),
                                             codes.ctypes.data, scales.ctypes.data)
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_read_intermediate")
        n = self.routing(stream)["num_rows"]
        return codes[:n], scales[:n]

    def set_timing(self, enable: bool):
        lib().afd_ffn_set_timing(self.plan, 1 if enable else 0)

    def kernel_times(self):
        ms = (c_float * len(KERNEL_NAMES))()
        rc = lib().afd_ffn_get_kernel_times(self.plan, ms)
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_get_kernel_times")
        return dict(zip(KERNEL_NAMES, list(ms)))

    def set_wait_limit(self, ns: int):
        rc = lib().afd_ffn_set_wait_limit(self.plan, int(ns))
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_set_wait_limit")

    def set_tiling(self, tiling: int):
        """0: default (1); 1: software-promoted block-FP8 GEMMs (any fp32 block scales); 2: W13
        on the block-scale MMA path, for inputs whose activation and W13 block scales are all
        powers of two (the first selection builds and checks the W13 factor images and
        synchronises the device; weights with other scales are refused)."""
        rc = lib().afd_ffn_set_tiling(self.plan, int(tiling))
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_set_tiling")

    def tiling(self, stream=None) -> int:
        """Tiling (1 or 2) the last layer call used."""
        t = c_int32(0)
        rc = lib().afd_ffn_get_tiling(self.plan, c_void_p(_stream_handle(stream)), ctypes.byref(t))
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_get_tiling")
        return t.value

    def inject_stall(self, enable: bool = True):
        lib().afd_ffn_inject_stall(self.plan, 1 if enable else 0)

    def set_combine_targets(self, accs: Optional[Sequence]):
        """Expert-parallel return path: the down projection adds each token's weighted rows
        into accs[m] (fp32 [capacity, hidden] per received slab, possibly tensors that view
        another GPU's memory) and the call stops after it; None restores the plan's own
        accumulators and the bf16 slab outputs. The owner finishes with combine_finalize."""
        if accs is None:
            rc = lib().afd_ffn_set_combine_targets(self.plan, None)
        else:
            if len(accs) != self.num_slabs:
                raise ValueError("expected %d accumulators" % self.num_slabs)
            cap, H = self.slab_capacity, self.shape.hidden
            for a in accs:
                if str(a.dtype) != "torch.float32":
                    raise ValueError("accumulators must be float32")
                if tuple(a.shape) != (cap, H):
                    raise ValueError(f"accumulator shape {tuple(a.shape)} != {(cap, H)}")
            table = (c_void_p * self.num_slabs)(*[_ptr(a, "accumulator") for a in accs])
            self._targets = accs            # the caller's buffers stay referenced while in use
            rc = lib().afd_ffn_set_combine_targets(self.plan, table)
        if rc != AFD_OK:
            raise AfdError(rc, "afd_ffn_set_combine_targets")


def combine_finalize(slabs: Sequence, counts, accs: Sequence, stream=None) -> None:
    """Owner side of the expert-parallel return path: after every FFN GPU's partial rows
    have been added into accs (fp32 [capacity, hidden] per slab), write y[m][t] =
    bf16(accs[m][t]) for t < counts[m] and clear those accumulator rows."""
    M = len(slabs)
    if len(accs) != M:
        raise ValueError("one accumulator per slab")
    cap, H = accs[0].shape
    descs = (SlabDesc * M)()
    for i, s in enumerate(slabs):
        descs[i] = SlabDesc(None, None, None, None, _ptr(s.y, "y"))
    table = (c_void_p * M)(*[_ptr(a, "accumulator") for a in accs])
    rc = lib().afd_combine_finalize(descs, M, int(cap), int(H), c_void_p(_ptr(counts, "counts")), table,
                                    c_void_p(_stream_handle(stream)))
    if rc != AFD_OK:
        raise AfdError(rc, "afd_combine_finalize")


def kernels_per_layer(layer: "FfnLayer") -> int:
    """Kernel launches one call of `layer` makes with its current tiling."""
    return lib().afd_ffn_kernels_per_layer(layer.plan)


def route_noalloc(shape, slabs: Sequence, counts, stream=None) -> dict:
    """Routing through afd_ffn_route_noalloc: the library allocates nothing; the output
    buffers below are allocated here, by the caller, with torch.

    For callers that cannot call cudaMalloc at step time (a serving engine whose memory
    pool already holds nearly all of HBM, a loop that must not stall on allocation).
    Returns CUDA tensors: sizes [4] (T, R, m-tiles, 0), counts [G], offsets [G+1],
    row_token / row_k / row_weight [max_rows], pos [M*cap*K], status [1].
    """
    import torch
    M = len(slabs)
    cap = slabs[0].topk_ids.shape[0]
    cfg = make_config(shape, M, cap)
    G = shape.num_local_experts + shape.has_shared_expert
    max_rows = M * cap * (min(shape.top_k, shape.num_local_experts) + shape.has_shared_expert)
    dev = slabs[0].topk_ids.device
    i32 = dict(dtype=torch.int32, device=dev)
    out = {
        "sizes": torch.zeros(4, **i32), "counts": torch.zeros(G, **i32),
        "offsets": torch.zeros(G + 1, **i32), "row_token": torch.zeros(max(max_rows, 1), **i32),
        "row_k": torch.zeros(max(max_rows, 1), **i32),
        "row_weight": torch.zeros(max(max_rows, 1), dtype=torch.float32, device=dev),
        "pos": torch.zeros(max(M * cap * shape.top_k, 1), **i32), "status": torch.zeros(1, **i32),
    }
    descs = (SlabDesc * M)()
    for i, s in enumerate(slabs):
        descs[i] = SlabDesc(_ptr(s.x, "x"), _ptr(s.x_scale, "x_scale"), _ptr(s.topk_ids, "topk_ids"),
                            _ptr(s.topk_weights, "topk_weights"), _ptr(s.y, "y"))
    P = lambda k: c_void_p(out[k].data_ptr())
    rc = lib().afd_ffn_route_noalloc(ctypes.byref(cfg), descs, c_void_p(_ptr(counts, "counts")), P("sizes"),
                                     P("counts"), P("offsets"), P("row_token"), P("row_k"),
                                     P("row_weight"), P("pos"), P("status"),
                                     c_void_p(_stream_handle(stream)))
    if rc != AFD_OK:
        raise AfdError(rc, "afd_ffn_route_noalloc")
    return out
