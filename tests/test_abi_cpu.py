"""The C-ABI library loads on a CPU-only host, exports every function that
include/moe.h declares, and rejects bad arguments on the host before any CUDA
call (no compute is launched here)."""
import ctypes

import pytest

moe = pytest.importorskip("combine_overlap_b200.moe")


def test_exports_every_declared_symbol():
    names = moe.declared_symbols()
    assert {"moe_route", "moe_permute", "moe_layer_forward", "moe_grouped_ffn", "moe_combine",
            "moe_workspace_size", "moe_get_status", "moe_status_string", "moe_num_sms"} <= set(names)
    lib = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_workspace_size_rules():
    ws = moe.workspace_size
    assert ws(256, 512, 1024, 8, 2) > 0
    assert ws(0, 512, 1024, 8, 2) == 0          # no tokens
    assert ws(256, 512, 1024, 8, 9) == 0        # k > E
    assert ws(256, 500, 1024, 8, 2) == 0        # d not a multiple of 256
    assert ws(256, 512, 1000, 8, 2) == 0        # f not a multiple of 128
    assert ws(256, 512, 1024, 300, 2) == 0      # E > 256
    assert ws(256, 512, 1024, 16, 9) == 0       # k > 8
    # grows with every dimension; the intermediates dominate
    base = ws(256, 512, 1024, 8, 2)
    for args in ((512, 512, 1024, 8, 2), (256, 1024, 1024, 8, 2), (256, 512, 2048, 8, 2),
                 (256, 512, 1024, 8, 4)):
        assert ws(*args) > base
    R = 4096 * 2
    assert ws(4096, 4096, 14336, 8, 2) >= R * 4096 * 2 + R * 14336 * 2   # y and h


def test_status_strings():
    for c in range(6):
        assert moe.status_string(c)


def test_cuda_error_reporting():
    assert isinstance(moe.last_cuda_error(), int)
    assert moe.cuda_error_string(0) == "no error"
    assert "illegal instruction" in moe.cuda_error_string(715)
    # host-side rejections are not CUDA errors: no CUDA detail is attached to them
    err = moe.MoEError(moe.MOE_ERR_INVALID, "call")
    assert err.cuda_error == 0 and "invalid argument" in str(err) and "cudaError" not in str(err)
    assert moe.status_string(4).startswith("a bounded device wait")


def _call_forward(args, mode=1, ws=0x1000, ws_bytes=1 << 40):
    return moe._lib.moe_layer_forward(ctypes.byref(args), mode, ctypes.c_void_p(ws), ws_bytes, None)


def _args(**kw):
    a = moe.LayerArgs(256, 512, 1024, 8, 2, 0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000,
                      0, 0, 0, 0, 0, 0, 1, 0, 0, None, None)
    for k_, v in kw.items():
        setattr(a, k_, v)
    return a


def test_host_side_argument_errors():
    # every one of these returns before the library touches the GPU
    assert _call_forward(_args(k=9)) == moe.MOE_ERR_INVALID
    assert _call_forward(_args(T=0)) == moe.MOE_ERR_INVALID
    assert _call_forward(_args(d=320)) == moe.MOE_ERR_UNSUPPORTED
    assert _call_forward(_args(x=0)) == moe.MOE_ERR_INVALID
    assert _call_forward(_args(out=0x6008)) == moe.MOE_ERR_INVALID      # misaligned
    assert _call_forward(_args(consumer_sms=-1)) == moe.MOE_ERR_INVALID
    assert _call_forward(_args(), mode=7) == moe.MOE_ERR_INVALID
    assert _call_forward(_args(), ws=0) == moe.MOE_ERR_WORKSPACE
    assert _call_forward(_args(), ws_bytes=1024) == moe.MOE_ERR_WORKSPACE
    assert moe._lib.moe_layer_forward(None, 1, None, 0, None) == moe.MOE_ERR_INVALID
    P = ctypes.c_void_p
    assert moe._lib.moe_route(P(0x1000), 16, 8, 0, P(0x2000), P(0x3000), None, P(0x4000), 1 << 30,
                              None) == moe.MOE_ERR_INVALID
    assert moe._lib.moe_route(P(0x1000), 16, 8, 2, P(0x2000), P(0x3000), None, None, 1 << 30,
                              None) == moe.MOE_ERR_WORKSPACE
    assert moe._lib.moe_combine(P(0x1000), P(0x2000), P(0x3000), 16, 512, 9, P(0x4000),
                                None) == moe.MOE_ERR_UNSUPPORTED


def test_tile_variant_rule():
    tv = moe.tile_variant
    # 256-row tiles on single CTAs from 256 rows per expert (T*k/E) up, else 128-row tiles
    assert tv(4096, 14336, 8, 2) == 3          # Mixtral-shaped: 1024 rows per expert
    assert tv(8192, 1408, 64, 6) == 3          # fine-grained: 768
    assert tv(1024, 2048, 8, 2) == 3           # exactly 256
    assert tv(1023, 2048, 8, 2) == 1           # just below
    assert tv(512, 2048, 32, 4) == 1           # 64
    # flags force a variant; ONE_CTA before CTA_PAIR before WIDE_CTA
    assert tv(4096, 14336, 8, 2, moe.SCHED_ONE_CTA) == 1
    assert tv(512, 2048, 32, 4, moe.SCHED_CTA_PAIR) == 2
    assert tv(512, 2048, 32, 4, moe.SCHED_WIDE_CTA) == 3
    assert tv(512, 2048, 32, 4, moe.SCHED_ONE_CTA | moe.SCHED_CTA_PAIR) == 1
    assert tv(512, 2048, 32, 4, moe.SCHED_CTA_PAIR | moe.SCHED_WIDE_CTA) == 2
    # other flags do not change the choice
    assert tv(4096, 14336, 8, 2, moe.SCHED_NO_JOIN | moe.SCHED_B_PER_ATOM) == 3
    assert tv(0, 14336, 8, 2) == 0
    assert set(moe.TILE_VARIANTS) == {1, 2, 3}


def test_ep_owner_host_side_argument_errors():
    # moe_ep_owner_forward refuses bad shapes and pointers before any CUDA call
    ws = moe.ep_owner_workspace_size
    assert ws(1000, 512, 256, 4, 2) > 0
    assert ws(0, 512, 256, 4, 2) > 0            # an owner may receive nothing
    assert ws(1000, 500, 256, 4, 2) == 0        # d not a multiple of 256
    assert ws(1000, 512, 256, 4, 9) == 0        # more ranks than MOE_MAX_EP_RANKS
    assert ws(1000, 512, 256, 64, 8) == 0       # W * El > 256 planning units
    assert ws(-1, 512, 256, 4, 2) == 0

    def args(**kw):
        a = moe.EpOwnerArgs()
        a.W, a.rank, a.N, a.d, a.f, a.El, a.k = 2, 0, 100, 512, 256, 4, 2
        a.x_recv, a.slot_recv, a.recv_counts = 0x1000, 0x2000, 0x3000
        a.W1, a.W3, a.W2 = 0x4000, 0x5000, 0x6000
        for r in range(2):
            a.home_y[r] = 0x10000 * (r + 1)
            a.home_arrive[r] = 0x20000 * (r + 1)
        for k_, v in kw.items():
            setattr(a, k_, v)
        return a

    def call(a, mode=1, wsb=1 << 40):
        return moe._lib.moe_ep_owner_forward(ctypes.byref(a), mode, ctypes.c_void_p(0x100000), wsb, None)

    assert call(args(W=0)) == moe.MOE_ERR_INVALID
    assert call(args(rank=2)) == moe.MOE_ERR_INVALID
    assert call(args(W=9)) == moe.MOE_ERR_UNSUPPORTED
    assert call(args(El=200)) == moe.MOE_ERR_UNSUPPORTED      # 400 planning units
    assert call(args(d=320)) == moe.MOE_ERR_UNSUPPORTED
    assert call(args(x_recv=0)) == moe.MOE_ERR_INVALID
    assert call(args(x_recv=0x1008)) == moe.MOE_ERR_INVALID   # misaligned
    assert call(args(), mode=5) == moe.MOE_ERR_INVALID
    a = args()
    a.home_y[1] = 0
    assert call(a) == moe.MOE_ERR_INVALID
    assert call(args(), wsb=1024) == moe.MOE_ERR_WORKSPACE
    assert moe._lib.moe_ep_owner_forward(None, 1, None, 0, None) == moe.MOE_ERR_INVALID
    P = ctypes.c_void_p
    hc = moe._lib.moe_ep_home_combine
    assert hc(P(0x1000), P(0x2000), P(0x3000), P(0x4000), 0, 512, 2, P(0x5000), P(0x6000), 0,
              None) == moe.MOE_ERR_INVALID
    assert hc(P(0x1000), P(0x2000), P(0x3000), P(0x4000), 16, 512, 9, P(0x5000), P(0x6000), 0,
              None) == moe.MOE_ERR_UNSUPPORTED
    assert hc(P(0x1000), P(0x2000), P(0x3000), P(0x4000), 16, 512, 2, P(0x5000), None, 0,
              None) == moe.MOE_ERR_INVALID


def test_debug_tokens_combined_rejects_bad_arguments_on_the_host():
    # argument checks come before any device call, so they hold without a GPU
    n = ctypes.c_int(-1)
    f = moe._lib.moe_debug_tokens_combined
    assert f(None, 256, 512, 1024, 8, 2, None, ctypes.byref(n)) == moe.MOE_ERR_INVALID          # no ws
    assert f(ctypes.c_void_p(0x1001), 256, 512, 1024, 8, 2, None, ctypes.byref(n)) == moe.MOE_ERR_INVALID  # misaligned
    assert f(ctypes.c_void_p(0x1000), 256, 512, 1024, 8, 2, None, None) == moe.MOE_ERR_INVALID   # no output
    assert f(ctypes.c_void_p(0x1000), 256, 500, 1024, 8, 2, None, ctypes.byref(n)) == moe.MOE_ERR_UNSUPPORTED  # d % 256
    assert f(ctypes.c_void_p(0x1000), 256, 512, 1024, 8, 9, None, ctypes.byref(n)) == moe.MOE_ERR_INVALID  # k > E
    assert n.value == -1
