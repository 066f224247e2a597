"""CPU-only checks of the C-ABI library: it loads, exports every declared symbol,
and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nsa.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(nsa_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def abi():
    from dynamic_block_sparse_scoring_b200 import build
    build.build()
    from dynamic_block_sparse_scoring_b200 import abi as a
    return a


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["nsa_score_blocks", "nsa_topk_select", "nsa_sparse_attn_fwd", "nsa_pool_kv",
                 "nsa_workspace_size", "nsa_status_string"]:
        assert want in names


def test_library_exports_every_declared_symbol(abi):
    lib = ctypes.CDLL(abi._LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_config_struct_layout_matches_header(abi):
    # 13 int32 + float + uint32, no padding
    assert ctypes.sizeof(abi.NsaConfig) == 15 * 4


def test_status_strings(abi):
    for code in range(6):
        assert abi.nsa_status_string(code).startswith(abi.STATUS[code])


def _cfg(abi, **kw):
    from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS
    return abi.config(WORKLOADS["tiny"], **kw)


def test_workspace_sizes(abi):
    from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS
    for name, wl in WORKLOADS.items():
        cfg = abi.config(wl)
        n = abi.nsa_workspace_size(cfg)
        nmin = abi.nsa_workspace_size_min(cfg)
        # the selected ids, when the call selects blocks
        want = wl.batch * wl.h_sel * wl.seqlen_q * wl.top_k * 4 if wl.branches & 2 else 0
        assert nmin >= want and nmin % 256 == 0 and n >= nmin, name
    # the 64k NSA prefill runs its selected branch block-major: index + bf16 partials
    wl = WORKLOADS["nsa64k"]
    n = abi.nsa_workspace_size(abi.config(wl))
    assert n >= wl.seqlen_q * wl.h_kv * wl.top_k * wl.group * wl.d_v * 2
    # decode runs the few-query kernel (keys as the MMA M dimension, partials + merge)
    wl = WORKLOADS["decode64x64k"]
    cfg = abi.config(wl)
    assert abi.nsa_attn_plan(cfg, True, abi.nsa_workspace_size(cfg)) == ("decode", 3)
    # 4 heads per group: the query-major kernel with each tile's keys split over CTAs
    cfg4 = abi.config(WORKLOADS["tiny"].with_(seqlen_q=1, seqlen_kv=900, q_pos0=899))
    assert abi.nsa_attn_plan(cfg4, True, abi.nsa_workspace_size(cfg4))[0] == "split-k"
    assert abi.nsa_attn_plan(cfg, True, abi.nsa_workspace_size_min(cfg))[0] == "query-major"
    assert abi.nsa_attn_plan(abi.config(WORKLOADS["nsa64k"]), True,
                             abi.nsa_workspace_size(abi.config(WORKLOADS["nsa64k"])))[0] == "block-major"
    assert abi.nsa_attn_plan(abi.config(WORKLOADS["moba32k"]), True, 0)[0] == "rowwise"
    # MoBA (selected branch alone, one head per unit, 512-key blocks): block-major over
    # 64-key sub-blocks; expand + 4 index kernels + block-major + merge, after the selection
    moba = abi.config(WORKLOADS["moba32k"])
    n = abi.nsa_workspace_size(moba)
    wl = WORKLOADS["moba32k"]
    slots = wl.top_k * (wl.sel_block // 64)
    assert n >= wl.seqlen_q * wl.h_q * slots * wl.d_v * 2
    assert abi.nsa_attn_plan(moba, True, n) == ("block-major", 8)
    assert abi.nsa_attn_plan(moba, True, abi.nsa_workspace_size_min(moba))[0] == "rowwise"


@pytest.mark.parametrize("bad,status", [
    (dict(h_q=3, h_kv=2), 1),          # h_q not a multiple of h_kv
    (dict(batch=0), 1),
    (dict(seqlen_kv=0), 1),
    (dict(q_pos0=1), 1),               # q_pos0 + Tq > Tkv
    (dict(flags=0), 1),
    (dict(flags=128 | 7), 1),          # unknown flag bit
    (dict(top_k=0), 1),
    (dict(window=0), 1),
    (dict(cmp_stride=0), 1),
    (dict(scale=float("nan")), 1),
    (dict(d_qk=96), 2),
    (dict(d_v=32), 2),
    (dict(sel_block=24), 2),
    (dict(top_k=33), 2),
    (dict(cmp_block=24, cmp_stride=16), 2),
    (dict(h_q=32, h_kv=1), 2),         # group of 32 heads
])
def test_invalid_configs_rejected_on_host(abi, bad, status):
    cfg = _cfg(abi, **bad)
    n = ctypes.c_size_t(0)
    assert abi.lib.nsa_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == status
    # the compute entry points validate before launching: no device is touched
    fake = 1 << 20
    assert abi.lib.nsa_pool_kv(ctypes.byref(cfg), fake, fake, fake, fake, fake, None) == status
    assert abi.lib.nsa_sparse_attn_fwd(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake,
                                       fake, fake, fake, fake, 1 << 30, None) == status


def test_null_and_misaligned_pointers_rejected(abi):
    cfg = _cfg(abi)
    L = abi.lib
    c = ctypes.byref(cfg)
    good, odd = 1 << 20, (1 << 20) + 8
    assert L.nsa_pool_kv(c, None, good, good, good, good, None) == 1
    assert L.nsa_pool_kv(c, odd, good, good, good, good, None) == 1
    assert L.nsa_score_blocks(c, good, good, None, None) == 1
    assert L.nsa_topk_select(c, good, good, None, None, None) == 1
    assert L.nsa_topk_select(c, None, None, None, good, None) == 1
    assert L.nsa_sparse_attn_fwd(c, good, good, good, good, good, good, good, good, None, None, 0,
                                 None) == 1
    # selecting inside needs a workspace of nsa_workspace_size() bytes
    assert L.nsa_sparse_attn_fwd(c, good, good, good, good, good, good, good, None, good, None, 0,
                                 None) == 3
    assert L.nsa_sparse_attn_fwd(c, good, good, good, good, good, good, good, None, good, good, 16,
                                 None) == 3
    assert L.nsa_workspace_size(c, None) == 1
    assert L.nsa_workspace_size(None, ctypes.byref(ctypes.c_size_t())) == 1


def test_binding_raises_on_error(abi):
    cfg = _cfg(abi, batch=0)
    with pytest.raises(abi.NsaError):
        abi.nsa_workspace_size(cfg)


def test_timing_read_without_a_timed_call(abi):
    L = abi.lib
    n = ctypes.c_int32(7)
    assert L.nsa_timing_read(0, None, None, ctypes.byref(n)) == 0
    assert n.value == 0
    assert L.nsa_timing_read(-1, None, None, ctypes.byref(n)) == 1
    assert L.nsa_timing_read(4, None, None, ctypes.byref(n)) == 1
    assert L.nsa_timing_read(0, None, None, None) == 1
    assert L.nsa_timing_enable(0) == 0
    assert abi.nsa_timing_read() == []


def test_sub_block_path_conditions(abi):
    """The per-head block-major path over 64-key sub-blocks takes the selected branch
    alone, one head per unit, >= 256 query rows, sel_block a multiple of 64 and at most
    64 sub-block slots per row; anything else keeps its previous organisation."""
    from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, BR_SEL, BR_WIN
    moba = WORKLOADS["moba32k"].with_(seqlen_q=1024, seqlen_kv=1024)

    def plan(wl):
        cfg = abi.config(wl)
        return abi.nsa_attn_plan(cfg, True, abi.nsa_workspace_size(cfg))

    assert plan(moba) == ("block-major", 8)
    assert plan(moba.with_(sel_block=128, top_k=32))[0] == "block-major"   # 64 slots
    assert plan(moba.with_(sel_block=1024, top_k=3))[0] == "block-major"   # 48 slots
    assert plan(moba.with_(sel_block=256, top_k=17))[0] == "rowwise"       # 68 slots
    assert plan(moba.with_(seqlen_q=255, q_pos0=769))[0] == "rowwise"      # few rows
    assert plan(moba.with_(sel_block=96))[0] == "rowwise"                  # not a multiple of 64
    assert plan(moba.with_(branches=BR_SEL | BR_WIN, window=128))[0] == "rowwise"
    # the workspace holds one partial row per sub-block slot
    small = abi.nsa_workspace_size(abi.config(moba.with_(sel_block=64, top_k=3)))
    assert abi.nsa_workspace_size(abi.config(moba)) > 4 * small


def test_append_kv_rejects_bad_arguments_on_host(abi):
    from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS
    wl = WORKLOADS["decode64x64k"]
    fake = 1 << 20
    L = abi.lib
    ok = abi.config(wl, seqlen_q=1, q_pos0=63)          # completes block 0 and compressed token 2
    # no new token, past the cache, null cache or source
    assert L.nsa_append_kv(abi.config(wl, seqlen_q=0, q_pos0=10), fake, fake, fake, fake, fake, fake,
                           fake, None) == 1
    assert L.nsa_append_kv(abi.config(wl, seqlen_q=2, q_pos0=wl.seqlen_kv - 1), fake, fake, fake, fake,
                           fake, fake, fake, None) == 1
    assert L.nsa_append_kv(ok, None, fake, fake, fake, fake, fake, fake, None) == 1
    assert L.nsa_append_kv(ok, fake, fake, None, fake, fake, fake, fake, None) == 1
    # a completed block needs kbar, a completed compressed token needs kcmp and vcmp
    assert L.nsa_append_kv(ok, fake, fake, fake, fake, None, fake, fake, None) == 1
    assert L.nsa_append_kv(ok, fake, fake, fake, fake, fake, None, fake, None) == 1
    # misaligned
    assert L.nsa_append_kv(ok, fake + 2, fake, fake, fake, fake, fake, fake, None) == 1


def test_bounded_wait_self_test_rejects_bad_limits_on_host(abi):
    assert abi.lib.nsa_check_bounded_wait(0, None) == 1
    assert abi.lib.nsa_check_bounded_wait(2_000_000_000, None) == 1
    assert abi.lib.nsa_set_wait_limit_ns(2_000_000_000) == 1


def test_score_variant_flags_validated_on_host(abi):
    from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS
    wl = WORKLOADS["tiny"]
    n = ctypes.c_size_t(0)
    L = abi.lib
    both = abi.config(wl, flags=wl.flags | abi.NSA_SCORE_PROB | abi.NSA_SCORE_CMP)
    assert L.nsa_workspace_size(ctypes.byref(both), ctypes.byref(n)) == 1
    no_cmp = abi.config(wl, flags=abi.NSA_BR_SEL | abi.NSA_SCORE_CMP)       # needs the compressed branch
    assert L.nsa_workspace_size(ctypes.byref(no_cmp), ctypes.byref(n)) == 1
    too_many_sinks = abi.config(wl, flags=wl.flags | (wl.top_k << abi.NSA_SINK_SHIFT))
    assert L.nsa_workspace_size(ctypes.byref(too_many_sinks), ctypes.byref(n)) == 1
    ok = abi.config(wl, flags=wl.flags | abi.NSA_SCORE_PROB | ((wl.top_k - 1) << abi.NSA_SINK_SHIFT))
    assert L.nsa_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == 0
    # the compressed-branch scores read kcmp: the plain entry points cannot serve them
    cmp_mode = abi.config(wl, flags=wl.flags | abi.NSA_SCORE_CMP)
    fake = 1 << 20
    assert L.nsa_score_blocks(ctypes.byref(cmp_mode), fake, fake, fake, None) == 1
    assert L.nsa_topk_select(ctypes.byref(cmp_mode), fake, fake, None, fake, None) == 1


def test_backward_validates_on_host(abi):
    from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS
    wl = WORKLOADS["tiny"]
    cfg = abi.config(wl)
    fake = 1 << 20
    L = abi.lib
    n = ctypes.c_size_t(0)
    assert L.nsa_bwd_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 0
    n_cmp = (wl.seqlen_kv - wl.cmp_block) // wl.cmp_stride + 1
    assert n.value >= n_cmp * (wl.d_qk + wl.d_v) * 4 * wl.h_kv
    args = [fake] * 12          # q, k, v, kcmp, vcmp, gates, idx, d_out, dq, dk, dv, dgates
    # the selected branch needs the forward's ids; gates need a gate gradient buffer
    a = list(args); a[6] = None
    assert L.nsa_sparse_attn_bwd(ctypes.byref(cfg), *a, fake, n.value, None) == 1
    a = list(args); a[11] = None
    assert L.nsa_sparse_attn_bwd(ctypes.byref(cfg), *a, fake, n.value, None) == 1
    # workspace too small
    assert L.nsa_sparse_attn_bwd(ctypes.byref(cfg), *args, fake, n.value - 256, None) == 3


def test_backward_limits_refused_on_host(abi):
    from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS
    fake = 1 << 20
    args = [fake] * 12
    for over in (dict(h_q=32, h_kv=1),                       # 32 heads share a unit
                 dict(d_qk=320),                             # wider than 256
                 dict(top_k=40)):                            # more kept blocks than the kernel holds
        cfg = abi.config(WORKLOADS["tiny"].with_(seqlen_q=256, seqlen_kv=256, **over))
        n = ctypes.c_size_t(0)
        abi.lib.nsa_bwd_workspace_size(ctypes.byref(cfg), ctypes.byref(n))
        assert abi.lib.nsa_sparse_attn_bwd(ctypes.byref(cfg), *args, fake, max(n.value, 1 << 20), None) == 2, over
