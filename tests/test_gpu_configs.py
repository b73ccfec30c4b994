"""GPU parity at the measured workloads' full sizes, in the launch
configuration the benchmark times (one moe_layer call).

The oracle cannot redo a whole 8192-token layer in f64 in seconds, so the
layer output is compared on a token sample computed one by one by the oracle:
tokens chosen so that every 128-row tile of every expert's block of GEMM rows
holds at least one checked pair (which also covers every 256-row tile and each
expert's ragged last tile), the last token, and a stride sample.  The
properties that hold at any size are checked on every token: the routing is
bit-exact against the oracle's selection on the GPU's own logits, and the
permutation is bit-exact against the oracle's counting sort.  Tokens whose
GPU selection differs from the oracle's f64 selection (near-ties) are counted
and printed.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402

STRIDE = {"decode_f32_t1": 1, "prefill_bf16_t512": 48, "routed_shared_t4096": 24, "skewed_zipf_t8192": 8,
          "q8_0_decode_t16": 16, "grouped_sigmoid_t512": 32, "q4k_q6k_decode_t16": 16,
          "gemm_h7168_i2048_e8_t2048": 16}


@pytest.mark.parametrize("name", workloads.CONFIG_ORDER)
def test_full_size_config(name):
    spec = workloads.CONFIGS[name]
    wl = workloads.make(spec)
    desc, w, x = _gpu.upload(wl)
    out = _gpu.run_layer(desc, w, x)
    logits, ids, tw, sg = _gpu.run_route(desc, w, x)
    L = oracle.from_workload(wl)

    # routing on every token: bit-exact against the oracle's selection of the GPU's logits
    gl = logits.cpu().numpy().astype(np.float64)
    ref_ids, ref_w = oracle.select(gl, spec.K, spec.renormalize, gating=spec.gating, n_groups=spec.n_groups,
                                   topk_groups=spec.topk_groups)
    gids = ids.cpu().numpy()
    assert np.array_equal(gids, ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) < 2e-6

    # permutation of every pair: bit-exact
    P = spec.T * spec.K
    counts = torch.empty(spec.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(spec.E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(P, dtype=torch.int32, device="cuda")
    pp = torch.empty(P, dtype=torch.int32, device="cuda")
    moe.permute(desc, ids.reshape(-1), counts, offsets, sp, pp)
    rc, ro, rs, rp = oracle.permute(gids, spec.E)
    assert np.array_equal(counts.cpu().numpy(), rc) and np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(sp.cpu().numpy(), rs) and np.array_equal(pp.cpu().numpy(), rp)

    # layer output: a pair in every 128-row tile of every expert, the last token, a stride sample
    stride = np.linspace(0, spec.T - 1, STRIDE[name]).round().astype(int).tolist()
    cover = _gpu.tile_cover_tokens(gids, spec.E) if spec.T > 1 else [0]
    tokens = sorted(set(stride) | set(cover) | {spec.T - 1})
    exp, flagged = _gpu.expected_layer(L, gids, tokens, gpu_logits=gl)
    got = _gpu.to_np(out)[tokens]
    err = _gpu.assert_close(got, exp, spec.act_dtype, name)
    print(f"\n{name}: {len(tokens)} tokens checked ({len(cover)} cover every 128-row tile), "
          f"{flagged} near-tie tokens flagged, max|gpu-oracle| = {err:.3e}")
