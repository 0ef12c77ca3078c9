"""GPU parity of the MoE layer at the Kimi-K2.5 shapes (384 experts, top-8,
hidden 7168, intermediate 2048; the paper's serving integration, App. D.1:
dispatch-quantise -> gate_up -> SwiGLU + requantise -> down -> combine),
through moesq_moe_layer on all T tokens, against the oracle layer on a
sample of tokens.

A token's output depends only on its own logits, activations and the static
per-expert global scales, so the oracle runs the sampled tokens alone with
the seeded weights of just the experts they touch.  The activation global
scales come from the oracle: gamma_a from the largest |x| of the batch,
gamma_h from the largest |h| of the sampled tokens' SwiGLU rows.

T = 4096 with Zipf routing takes the paths the prefill bench takes: 128-row
token tiles in both GEMMs and the count / scan / scatter routing kernels
(T > 512); T = 1 takes 64-row tiles and the single-CTA routing finish."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from gpu_cases import oracle_pack_experts, pack_gpu_generated, to_dev, to_np

pytestmark = pytest.mark.gpu

E, K_TOP, H, I = 384, 8, 7168, 2048
SEED = 41


@pytest.fixture(scope="module")
def kimi_layer_weights(cuda_lib):
    m = cuda_lib
    pw_gu = pack_gpu_generated(m, SEED, 0, E, 2 * I, H, chunk=4)
    pw_dn = pack_gpu_generated(m, SEED, 1, E, H, I, chunk=8)
    return pw_gu, pw_dn


def _sample_tokens(rt, T, k):
    """Token 0, the last token, and the first tokens routed to the heaviest
    and to the lightest used expert."""
    ids = rt.topk_ids
    used = np.nonzero(rt.counts)[0]
    heavy = int(used[np.argmax(rt.counts[used])])
    light = int(used[np.argmin(rt.counts[used])])
    toks = {0, T - 1}
    for e in (heavy, light):
        toks.add(int(np.nonzero((ids == e).any(axis=1))[0][0]))
    return np.array(sorted(toks), np.int64)


@pytest.mark.parametrize("T,routing", [(1, "uniform"), (4096, "zipf")])
def test_kimi_layer_sampled_tokens(cuda_lib, kimi_layer_weights, T, routing):
    torch = pytest.importorskip("torch")
    m = cuda_lib
    pw_gu, pw_dn = kimi_layer_weights
    x = S.activations_bf16_np(SEED + T, T, H)
    lg = S.zipf_logits_np(SEED + T, T, E) if routing == "zipf" else S.uniform_logits_np(SEED + T, T, E)

    # oracle on the token sample
    rt_all = O.route(lg, K_TOP)
    toks = _sample_tokens(rt_all, T, K_TOP)
    xs, lgs = x[toks], lg[toks]
    used = np.nonzero(O.route(lgs, K_TOP).counts)[0]
    pk_gu = oracle_pack_experts(SEED, 0, E, 2 * I, H, used)
    pk_dn = oracle_pack_experts(SEED, 1, E, H, I, used)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    _, mid = O.moe_layer(xs, lgs, K_TOP, pk_gu, pk_dn, ga, np.ones(E, np.float32), keep=True)
    gh = np.full(E, O.global_scale(float(np.abs(mid["h"]).max())), np.float32)
    ref = O.moe_layer(xs, lgs, K_TOP, pk_gu, pk_dn, ga, gh)

    # CUDA layer on all T tokens
    ws = torch.empty(m.moesq_layer_workspace_bytes(T, K_TOP, E, H, I), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    m.moesq_moe_layer(to_dev(x), to_dev(lg), T, K_TOP, pw_gu, pw_dn, to_dev(ga), to_dev(gh), out, ws)
    st, word = m.moesq_get_device_error()
    assert st == 0, hex(word)
    got = to_np(out)[toks]
    for j in range(toks.size):
        o = S.bf16_bits_to_f32_np(got[j]).astype(np.float64)
        r = S.bf16_bits_to_f32_np(ref[j]).astype(np.float64)
        rel = np.abs(o - r).max() / np.abs(r).max()
        assert rel <= 2e-2, (T, int(toks[j]), rel, np.abs(o - r).mean() / np.abs(r).mean())
