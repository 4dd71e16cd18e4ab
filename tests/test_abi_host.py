"""The C-ABI library on the host: it loads, exports every declared entry point, and
validates arguments without touching a GPU."""
import ctypes
import os
import re

import pytest
import torch

import workloads as W
from attention_ffn_disaggregated_b200 import ffn

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "afd_ffn.h")


def declared_functions():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^AFD_API\s+[\w\s\*]+?\b(afd_\w+)\s*\(", txt, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("afd_ffn_plan", "afd_ffn_layer", "afd_ffn_destroy"):
        assert required in names
    assert len(names) >= 14


def test_library_exports_every_declared_symbol():
    L = ffn.lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def _cfg(**kw):
    base = dict(hidden=256, intermediate=128, num_experts_global=8, expert_begin=0,
                num_local_experts=8, has_shared_expert=0, top_k=2, num_slabs=2, slab_capacity=32)
    base.update(kw)
    return ffn.Config(**base)


@pytest.mark.parametrize("kw,code", [
    ({}, 0),
    ({"hidden": 0}, 1), ({"hidden": 200}, 1), ({"intermediate": 64}, 1),
    ({"hidden": 384}, 2),                         # multiple of 128, not of 256
    ({"num_experts_global": 0}, 1), ({"expert_begin": -1}, 1),
    ({"expert_begin": 4, "num_local_experts": 5}, 1),
    ({"has_shared_expert": 2}, 1),
    ({"num_local_experts": 0, "has_shared_expert": 0}, 1),
    ({"num_local_experts": 0, "has_shared_expert": 1}, 0),
    ({"top_k": 0}, 1), ({"top_k": 9}, 1),
    ({"num_experts_global": 64, "num_local_experts": 64, "top_k": 33}, 2),
    ({"num_slabs": 0}, 1), ({"num_slabs": 129}, 2), ({"slab_capacity": 0}, 1),
    ({"slab_capacity": 1 << 24}, 2),
    ({"num_experts_global": 2048, "num_local_experts": 1024, "has_shared_expert": 1}, 2),
    ({"hidden": 16640}, 2), ({"intermediate": 16512}, 2),   # above 128 quantisation blocks
])
def test_check_config_codes(kw, code):
    c = _cfg(**kw)
    assert ffn.lib().afd_ffn_check_config(ctypes.byref(c)) == code


def test_check_config_null():
    assert ffn.lib().afd_ffn_check_config(None) == 1


def test_every_benchmark_config_is_valid():
    for wl in list(W.CONFIGS.values()) + W.sweep_workloads():
        c = ffn.make_config(wl.shape, wl.num_slabs, wl.slab_capacity)
        assert ffn.check_config(c) == 0, wl.name


def test_destroy_null_is_noop():
    ffn.lib().afd_ffn_destroy(None)


def test_null_arguments_rejected():
    L = ffn.lib()
    c = _cfg()
    w = ffn.Weights(None, None, None, None)
    h = ctypes.c_void_p()
    assert L.afd_ffn_plan(ctypes.byref(c), ctypes.byref(w), None) == 1
    assert L.afd_ffn_plan(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == 1
    assert h.value is None
    assert L.afd_ffn_layer(None, None, None, None) == 1
    assert L.afd_ffn_get_status(None, None, None) == 1
    assert L.afd_ffn_set_timing(None, 1) == 1
    assert L.afd_ffn_get_info(None, None) == 1
    assert L.afd_ffn_kernels_per_layer(None) == -1
    assert L.afd_status_string(6) == b"AFD_ERR_TIMEOUT"


def test_misaligned_weights_rejected():
    L = ffn.lib()
    c = _cfg()
    w = ffn.Weights(0x1001, 0x2000, 0x3000, 0x4000)
    h = ctypes.c_void_p()
    assert L.afd_ffn_plan(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == 1


@pytest.mark.skipif(torch.cuda.is_available(), reason="host without a GPU only")
def test_plan_without_gpu_is_unsupported():
    L = ffn.lib()
    c = _cfg()
    w = ffn.Weights(0x1000, 0x2000, 0x3000, 0x4000)
    h = ctypes.c_void_p()
    assert L.afd_ffn_plan(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == 2
    assert h.value is None


def test_binding_refuses_host_tensors():
    """The binding hands only CUDA tensors' addresses to the library: a host tensor
    (which the kernels would read as a device address) is refused before any call."""
    import torch
    from attention_ffn_disaggregated_b200.ffn import _ptr
    assert _ptr(None) is None
    with pytest.raises(ValueError, match="w13 must be a CUDA tensor"):
        _ptr(torch.zeros(16, dtype=torch.uint8), "w13")


def test_return_path_entry_points_validate_arguments():
    """afd_ffn_set_combine_targets and afd_combine_finalize refuse bad arguments before
    touching a GPU (NULL plan or tables, misaligned or NULL buffers, sizes out of range)."""
    L = ffn.lib()
    assert L.afd_ffn_set_combine_targets(None, None) == 1
    slabs = (ffn.SlabDesc * 2)()
    for i in range(2):
        slabs[i] = ffn.SlabDesc(None, None, None, None, 0x10000 + 0x1000 * i)
    acc = (ctypes.c_void_p * 2)(0x20000, 0x30000)
    counts = ctypes.c_void_p(0x40000)
    fin = L.afd_combine_finalize
    assert fin(None, 2, 8, 256, counts, acc, None) == 1                  # no slabs
    assert fin(slabs, 2, 8, 256, None, acc, None) == 1                   # no counts
    assert fin(slabs, 2, 8, 256, counts, None, None) == 1                # no accumulators
    assert fin(slabs, 0, 8, 256, counts, acc, None) == 1                 # no slabs to finish
    assert fin(slabs, 129, 8, 256, counts, acc, None) == 1               # above the slab limit
    assert fin(slabs, 2, 0, 256, counts, acc, None) == 1                 # zero capacity
    assert fin(slabs, 2, 8, 384, counts, acc, None) == 1                 # hidden not a multiple of 256
    bad = (ctypes.c_void_p * 2)(0x20000, 0x30004)                        # misaligned accumulator
    assert fin(slabs, 2, 8, 256, counts, bad, None) == 1
    nul = (ctypes.c_void_p * 2)(0x20000, None)
    assert fin(slabs, 2, 8, 256, counts, nul, None) == 1
    slabs[1] = ffn.SlabDesc(None, None, None, None, 0x10008)              # misaligned output rows
    assert fin(slabs, 2, 8, 256, counts, acc, None) == 1
