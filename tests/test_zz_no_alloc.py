"""mla_decode_fwd_noalloc (fixed scratch inside the library, planner inside the
call) against mla_decode_fwd (caller workspace and metadata) on the same
inputs, through the C ABI.  Collected last so it also runs after every other
GPU test in the same process."""
import pytest
import torch

from mla_paged_kv_03_b200 import binding as B
from mla_paged_kv_03_b200 import workloads as W
from parity_util import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu


def _to_dev(case):
    dev = torch.device("cuda")
    return (case.q.to(dev), case.kcache.to(dev), case.block_table.to(dev),
            case.cache_seqlens.to(dev))


def _with_workspace(case, q, kc, bt, sl):
    meta, ns, parts = B.mla_get_metadata(sl, case.s_q * case.h_q, 1)
    return B.mla_decode_fwd(q, kc, bt, sl, case.d_v, meta, ns, parts, causal=case.causal,
                            softmax_scale=case.softmax_scale)


def _noalloc(case, q, kc, bt, sl):
    return B.mla_decode_fwd_noalloc(q, kc, bt, sl, case.d_v, causal=case.causal,
                                    softmax_scale=case.softmax_scale)


def test_noalloc_matches_workspace_path_on_consecutive_calls():
    # 32 rows per sequence (page kernel), 128 rows (CTA-pair kernel), d_v 576
    # (1-CTA kernel, whose partials are 576 wide), then the first case again:
    # each call reuses the same scratch array.
    cases = [
        W.make_dense(W.lengths_loguniform(24, 64, 6000, seed=5), 2, 16, seed=5, name="mem"),
        W.make_dense(W.lengths_uniform(3, 500, 3000, seed=6), 1, 128, seed=6, q_std=0.5,
                     k_std=0.5, name="h128"),
        W.make_dense(W.lengths_uniform(5, 100, 4000, seed=8), 1, 64, seed=8, d_v=576,
                     name="dv576"),
    ]
    cases.append(cases[0])
    for case in cases:
        t = _to_dev(case)
        ref_o, ref_l = _with_workspace(case, *t)
        out, lse = _noalloc(case, *t)
        torch.cuda.synchronize()
        assert B.device_status() == 0
        assert_out_close(out, ref_o.double().cpu().numpy())
        assert_lse_close(lse, ref_l.double().cpu().numpy())


def test_noalloc_rejects_problem_beyond_fixed_scratch():
    case = W.make_dense([64] * 256, 1, 128, seed=7)
    t = _to_dev(case)
    with pytest.raises(B.MLAError) as e:
        _noalloc(case, *t)
    assert e.value.code == B.MLA_ERR_INVALID_ARG
    assert "scratch" in str(e.value)
    assert B.mla_noalloc_scratch_bytes() == 32 << 20
