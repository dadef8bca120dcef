"""Host-side checks of the C ABI that need no GPU: the library loads, every function
declared in include/gptq_b200.h is exported, and argument validation rejects bad
calls before anything is enqueued."""

import ctypes

import pytest

from post_weight_quantization_14_b200 import gptq as G


def test_library_exports_every_declared_function():
    L = G.lib()
    names = G.header_functions()
    assert len(names) >= 16
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    # every declared function has a ctypes signature in the binding
    assert set(names) <= set(G._SIGS)


def test_default_config_and_strings():
    c = G.make_config()
    assert (c.bits, c.group_size, c.sym, c.block_size, c.desc_act) == (4, 128, 0, 128, 0)
    assert c.damp_rel == pytest.approx(0.01)
    L = G.lib()
    assert L.gptq_status_string(G.GPTQ_ERR_NOT_PD) == b"GPTQ_ERR_NOT_PD"
    assert L.gptq_status_string(99) == b"GPTQ_ERR_UNKNOWN"
    assert L.gptq_version() >= 100


def test_workspace_queries_are_positive_and_grow():
    L = G.lib()
    c = G.make_config()
    small = L.gptq_quantize_workspace_bytes(256, 256, ctypes.byref(c))
    big = L.gptq_quantize_workspace_bytes(4096, 4096, ctypes.byref(c))
    assert 0 < small < big
    assert L.gptq_prepare_hinv_workspace_bytes(200) > 200 * 200 * 4
    assert L.gptq_hessian_workspace_bytes(100, 64, G.GPTQ_BF16) >= 64 * 128 * 2
    assert L.gptq_hessian_workspace_bytes(100, 64, G.GPTQ_F32) >= 2 * 64 * 128 * 4
    assert L.gptq_hessian_workspace_bytes(0, 64, G.GPTQ_F32) == 0


def _fake(n=1):
    # host addresses are never dereferenced: validation fails before any CUDA call
    return ctypes.c_void_p(0x1000 * n)


@pytest.mark.parametrize("field,value,status", [
    ("bits", 5, G.GPTQ_ERR_INVALID_ARG),
    ("bits", 1, G.GPTQ_ERR_INVALID_ARG),
    ("group_size", 48, G.GPTQ_ERR_INVALID_ARG),
    ("group_size", 8, G.GPTQ_ERR_INVALID_ARG),
    ("group_size", 256, G.GPTQ_ERR_INVALID_ARG),
    ("block_size", 64, G.GPTQ_ERR_INVALID_ARG),
    ("sym", 2, G.GPTQ_ERR_INVALID_ARG),
    ("desc_act", 1, G.GPTQ_ERR_INVALID_ARG),     # the natural-order loop; act order has its own call
    ("desc_act", 3, G.GPTQ_ERR_INVALID_ARG),
    ("damp_rel", -1.0, G.GPTQ_ERR_INVALID_ARG),
    ("damp_rel", float("nan"), G.GPTQ_ERR_INVALID_ARG),
])
def test_quantize_rejects_bad_config(field, value, status):
    c = G.make_config()
    setattr(c, field, value)
    L = G.lib()
    st = L.gptq_quantize_layer(_fake(1), _fake(2), 64, 64, ctypes.byref(c), _fake(3), _fake(4), _fake(5),
                               None, _fake(6), 1 << 30, None)
    assert st == status
    assert L.gptq_last_error()


def test_quantize_rejects_bad_shapes_and_pointers():
    L = G.lib()
    c = G.make_config()
    args = lambda W, d_out, d_in, qz: L.gptq_quantize_layer(W, _fake(2), d_out, d_in, ctypes.byref(c), _fake(3),
                                                            _fake(4), qz, None, _fake(6), 1 << 40, None)
    assert args(None, 64, 64, _fake(5)) == G.GPTQ_ERR_INVALID_ARG
    assert args(_fake(1), 64, 60, _fake(5)) == G.GPTQ_ERR_INVALID_ARG      # d_in % 8
    assert args(_fake(1), 0, 64, _fake(5)) == G.GPTQ_ERR_INVALID_ARG
    assert args(_fake(1), 64, 64, None) == G.GPTQ_ERR_INVALID_ARG          # asym needs qzeros
    c.sym = 1
    assert args(_fake(1), 64, 64, _fake(5)) == G.GPTQ_ERR_INVALID_ARG      # sym forbids qzeros
    # workspace too small
    c.sym = 0
    st = L.gptq_quantize_layer(_fake(1), _fake(2), 64, 64, ctypes.byref(c), _fake(3), _fake(4), _fake(5), None,
                               _fake(6), 16, None)
    assert st == G.GPTQ_ERR_WORKSPACE


def test_hessian_and_hinv_reject_bad_args():
    L = G.lib()
    assert L.gptq_hessian_accumulate(None, 0, 10, 64, _fake(2), 0, _fake(3), 1 << 30, None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_hessian_accumulate(_fake(1), 7, 10, 64, _fake(2), 0, _fake(3), 1 << 30, None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_hessian_accumulate(_fake(1), 0, 10, 66, _fake(2), 0, _fake(3), 1 << 30, None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_hessian_accumulate(_fake(1), 0, 10, 64, _fake(2), 0, _fake(3), 8, None) == G.GPTQ_ERR_WORKSPACE
    bad = ctypes.c_int64(0)
    lam = ctypes.c_float(0)
    assert L.gptq_prepare_hinv(None, 64, 0.01, _fake(2), _fake(3), 1 << 30, ctypes.byref(bad), ctypes.byref(lam),
                               None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_prepare_hinv(_fake(1), 64, -0.5, _fake(2), _fake(3), 1 << 30, None, None,
                               None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_prepare_hinv(_fake(1), 64, 0.01, _fake(2), _fake(3), 64, None, None, None) == G.GPTQ_ERR_WORKSPACE


def test_pack_and_dequant_reject_bad_args():
    L = G.lib()
    assert L.gptq_pack_int(_fake(1), 4, 8, 5, 0, _fake(2), None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_pack_int(_fake(1), 4, 8, 4, 2, _fake(2), None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_pack_int(_fake(1), 0, 8, 4, 0, _fake(2), None) == G.GPTQ_ERR_INVALID_ARG
    c = G.make_config(sym=True)
    assert L.gptq_dequant(_fake(1), _fake(2), _fake(3), 4, 8, ctypes.byref(c), _fake(4), None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_selftest_bounded_wait(10 ** 12, None) == G.GPTQ_ERR_INVALID_ARG


def test_product_path_has_no_cpu_fallback():
    # the binding refuses host tensors instead of computing on the CPU
    import torch
    W = torch.zeros(8, 8)
    with pytest.raises(ValueError):
        G._ptr(W)


def test_act_order_entry_points_validate_arguments():
    L = G.lib()
    c = G.make_config(desc_act=0)
    q = lambda cfg, perm=_fake(7), g_idx=_fake(8), ws=1 << 40: L.gptq_quantize_layer_act_order(
        _fake(1), _fake(2), perm, 64, 64, ctypes.byref(cfg), _fake(3), _fake(4), _fake(5), g_idx, None, _fake(6),
        ws, None)
    assert q(c) == G.GPTQ_ERR_INVALID_ARG                      # desc_act 0 belongs to gptq_quantize_layer
    c.desc_act = 1
    assert q(c, perm=None) == G.GPTQ_ERR_INVALID_ARG
    assert q(c, g_idx=None) == G.GPTQ_ERR_INVALID_ARG
    assert q(c, ws=16) == G.GPTQ_ERR_WORKSPACE
    c.desc_act = 5
    assert q(c) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_act_order(_fake(1), 64, 0, _fake(2), _fake(3), None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_act_order(_fake(1), 64, 3, _fake(2), _fake(3), None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_act_order(_fake(1), 0, 1, _fake(2), _fake(3), None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_act_sum_accumulate(_fake(1), G.GPTQ_F32, 10, 60, _fake(2), 0, None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_act_sum_accumulate(_fake(1), 7, 10, 64, _fake(2), 0, None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_prepare_hinv_permuted(_fake(1), None, 64, 0.01, _fake(2), _fake(3), 1 << 40, None, None,
                                        None) == G.GPTQ_ERR_INVALID_ARG
    assert L.gptq_dequant_g_idx(_fake(1), _fake(2), _fake(3), None, 8, 64, ctypes.byref(G.make_config()), _fake(4),
                                None) == G.GPTQ_ERR_INVALID_ARG


def test_act_order_workspace_covers_permuted_copies():
    L = G.lib()
    plain = L.gptq_quantize_workspace_bytes(4096, 4096, ctypes.byref(G.make_config()))
    act = L.gptq_quantize_workspace_bytes(4096, 4096, ctypes.byref(G.make_config(desc_act=1)))
    # a permuted copy of W (fp32) and of the packed 4-bit codes, plus the inverse permutation
    assert act - plain >= 4096 * 4096 * 4 + 4096 * 4096 // 2 + 4096 * 4


def test_dequant_gemm_validates_arguments():
    L = G.lib()
    call = lambda cfg, M=16, d_out=64, d_in=128, qz=_fake(4): L.gptq_dequant_gemm(
        _fake(1), M, _fake(2), _fake(3), qz, d_out, d_in, ctypes.byref(cfg), _fake(5), None)
    c = G.make_config(4, 128, False)
    assert call(c, d_in=96) == G.GPTQ_ERR_INVALID_ARG            # d_in % 64
    assert call(c, d_out=60) == G.GPTQ_ERR_INVALID_ARG           # d_out % 8
    assert call(c, M=0) == G.GPTQ_ERR_INVALID_ARG
    assert call(c, qz=None) == G.GPTQ_ERR_INVALID_ARG            # asymmetric needs qzeros
    assert call(G.make_config(3, 128, False)) == G.GPTQ_ERR_UNSUPPORTED   # 3-bit codes straddle words
    assert call(G.make_config(4, 32, False)) == G.GPTQ_ERR_UNSUPPORTED    # groups narrower than a K tile
    assert call(G.make_config(4, 128, False, desc_act=1)) == G.GPTQ_ERR_UNSUPPORTED


def test_binding_checks_act_order_tensor_types_before_any_call():
    import torch
    d = 64
    with pytest.raises(ValueError):
        G.gptq_act_order(torch.zeros(d, dtype=torch.float32), 1, torch.zeros(d, dtype=torch.int32),
                         torch.zeros(d, dtype=torch.int32))
    with pytest.raises(ValueError):
        G.gptq_act_order(torch.zeros(d, dtype=torch.float64), 1, torch.zeros(d, dtype=torch.int64),
                         torch.zeros(d, dtype=torch.int32))
    with pytest.raises(ValueError):
        G.gptq_prepare_hinv_permuted(torch.zeros((d, d)), torch.zeros(d, dtype=torch.int64), torch.zeros((d, d)))
    with pytest.raises(ValueError):
        G.gptq_dequant_g_idx(None, None, None, torch.zeros(d, dtype=torch.int64), 8, d, G.make_config(),
                             torch.zeros((8, d)))


def test_shared_input_checks_shapes_before_any_call():
    import torch
    X = torch.zeros((16, 64))
    with pytest.raises(ValueError):
        G.quantize_layers_shared_input([torch.zeros((8, 64)), torch.zeros((8, 32))], X)
    with pytest.raises(ValueError):
        G.quantize_layers_shared_input([torch.zeros((8, 64))], torch.zeros((16, 48)))
    assert G.quantize_layers_shared_input([], X) == []


def test_stage_wrappers_check_dtypes_and_shapes_before_any_call():
    """A wrong dtype or size must be refused in the binding: the C side sees only pointers
    and sizes, so it would read or write out of range on the device."""
    import torch
    d_out, d_in = 64, 128
    cfg = G.make_config(4, 128, False)
    qw = torch.zeros(((d_in * 4 + 31) // 32, d_out), dtype=torch.int32)
    sc = torch.zeros((1, d_out), dtype=torch.float16)
    qz = torch.zeros((1, (d_out * 4 + 31) // 32), dtype=torch.int32)
    es = torch.zeros((d_out,), dtype=torch.float32)
    W = torch.zeros((d_out, d_in), dtype=torch.float32)
    U = torch.zeros((d_in, d_in), dtype=torch.float32)
    bad = [
        (W.to(torch.bfloat16), U, qw, sc, qz, es),                      # bf16 W
        (W.half(), U, qw, sc, qz, es),                                  # fp16 W
        (W, torch.zeros((d_in - 8, d_in - 8)), qw, sc, qz, es),         # U of the wrong size
        (W, U.double(), qw, sc, qz, es),                                # fp64 U
        (W, U, qw[:-1], sc, qz, es),                                    # qweight too short
        (W, U, qw, sc.float(), qz, es),                                 # fp32 scales
        (W, U, qw, sc, None, es),                                       # asymmetric without qzeros
        (W, U, qw, sc, qz, torch.zeros((d_out - 1,))),                  # err_sq too short
    ]
    for args in bad:
        with pytest.raises(ValueError):
            G.gptq_quantize_layer(args[0], args[1], cfg, *args[2:])
    with pytest.raises(ValueError):
        G.gptq_prepare_hinv(torch.zeros((d_in, d_in)), torch.zeros((d_in, d_in - 8)))
    with pytest.raises(ValueError):
        G.gptq_prepare_hinv(torch.zeros((d_in, d_in), dtype=torch.float64), torch.zeros((d_in, d_in)))
    with pytest.raises(ValueError):
        G.gptq_dequant(qw, sc, qz, d_out, d_in, cfg, torch.zeros((d_out, d_in), dtype=torch.float16))
    with pytest.raises(ValueError):
        G.gptq_pack_int(torch.zeros((4, 8), dtype=torch.int32), 4, 0, torch.zeros((4, 1), dtype=torch.int32))
    with pytest.raises(ValueError):
        G.gptq_pack_int(torch.zeros((4, 8), dtype=torch.uint8), 4, 0, torch.zeros((4, 2), dtype=torch.int32))


def test_whole_layer_calls_refuse_arguments_that_conflict_with_the_buffers():
    from types import SimpleNamespace
    cfg = G.make_config(3, 64, True, 128, 0.02)
    bufs = SimpleNamespace(cfg=cfg)
    assert G._resolve_config(bufs, None, None, None, None, None) is cfg
    assert G._resolve_config(bufs, 3, 64, True, 0.02, 0) is cfg
    for kw in (dict(bits=4), dict(group_size=128), dict(sym=False), dict(damp_rel=0.01), dict(desc_act=1)):
        args = dict(bits=None, group_size=None, sym=None, damp_rel=None, desc_act=None)
        args.update(kw)
        with pytest.raises(ValueError):
            G._resolve_config(bufs, **args)
    d = G._resolve_config(None, None, None, None, None, None)
    assert (d.bits, d.group_size, d.sym, d.desc_act) == (4, 128, 0, 0)
    e = G._resolve_config(None, 2, 32, None, None, 2)
    assert (e.bits, e.group_size, e.sym, e.desc_act) == (2, 32, 0, 2)


def test_gptq2d_entry_validates_before_any_call():
    L = G.lib()
    ws = L.gptq_2d_workspace_bytes(64, 64, 1)
    assert ws >= 64 * 64 * 8
    assert L.gptq_2d_workspace_bytes(200, 150, 3) >= 200 * 200 * 8 + 3 * 200 * 150 * 8
    assert L.gptq_2d_workspace_bytes(0, 5, 1) == 0
    ok = lambda m=8, n=8, b=1, X=_fake(1), Z=_fake(4), wsb=1 << 30: L.gptq_2d_round(X, m, n, b, _fake(2), _fake(3), Z,
                                                                                     _fake(5), wsb, None)
    assert ok(m=0) == G.GPTQ_ERR_INVALID_ARG
    assert ok(n=20000) == G.GPTQ_ERR_INVALID_ARG
    assert ok(b=0) == G.GPTQ_ERR_INVALID_ARG
    assert ok(X=None) == G.GPTQ_ERR_INVALID_ARG
    assert ok(X=ctypes.c_void_p(0x1004)) == G.GPTQ_ERR_INVALID_ARG      # misaligned fp64
    assert ok(wsb=16) == G.GPTQ_ERR_WORKSPACE
