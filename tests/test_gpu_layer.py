"""GPU parity of the MoE layer (route -> dispatch-quantise -> gate_up ->
SwiGLU + requantise -> down -> combine) against the oracle layer:
max |out - out_ref| / max |out_ref| <= 2e-2."""
import numpy as np
import pytest

import layouts as L
import oracle as O
import synthetic as S
from gpu_cases import pack_gpu_from_np, to_dev, to_np, weights_np

pytestmark = pytest.mark.gpu


def _layer_case(m, E, k, H, I, T, seed, zipf=False):
    torch = pytest.importorskip("torch")
    wgu = weights_np(seed, 0, E, 2 * I, H)
    wdn = weights_np(seed, 1, E, H, I)
    pk_gu, pk_dn = O.pack_weights(wgu), O.pack_weights(wdn)
    x = S.activations_bf16_np(seed, T, H)
    lg = S.zipf_logits_np(seed, T, E) if zipf else S.uniform_logits_np(seed, T, E)
    ga, gh = O.calibrate_layer(x, lg, k, pk_gu, pk_dn)
    ref = O.moe_layer(x, lg, k, pk_gu, pk_dn, ga, gh)
    pw_gu, pw_dn = pack_gpu_from_np(m, wgu), pack_gpu_from_np(m, wdn)
    ws = torch.empty(m.moesq_layer_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    m.moesq_moe_layer(to_dev(x), to_dev(lg), T, k, pw_gu, pw_dn, to_dev(ga), to_dev(gh), out, ws)
    st, word = m.moesq_get_device_error()
    assert st == 0, hex(word)
    return to_np(out), ref, (x, lg, ga, gh, pw_gu, pw_dn, ws, pk_gu, pk_dn)


def _rel(out, ref):
    o = S.bf16_bits_to_f32_np(out).astype(np.float64)
    r = S.bf16_bits_to_f32_np(ref).astype(np.float64)
    return np.abs(o - r).max() / np.abs(r).max(), np.abs(o - r).mean() / np.abs(r).mean()


def test_layer_tiny(cuda_lib):
    out, ref, _ = _layer_case(cuda_lib, E=8, k=2, H=512, I=256, T=64, seed=3)
    rel, mean_rel = _rel(out, ref)
    assert rel <= 2e-2, (rel, mean_rel)


def test_layer_30b_class_shapes(cuda_lib):
    out, ref, _ = _layer_case(cuda_lib, E=128, k=8, H=2048, I=768, T=24, seed=5)
    rel, mean_rel = _rel(out, ref)
    assert rel <= 2e-2, (rel, mean_rel)


def test_layer_zipf_routing(cuda_lib):
    out, ref, _ = _layer_case(cuda_lib, E=32, k=4, H=512, I=256, T=160, seed=7, zipf=True)
    rel, mean_rel = _rel(out, ref)
    assert rel <= 2e-2, (rel, mean_rel)


def test_layer_host_entry_matches_device_entry(cuda_lib):
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, k, H, I, T = 8, 2, 512, 256, 40
    out, ref, (x, lg, ga, gh, pw_gu, pw_dn, _, _, _) = _layer_case(m, E, k, H, I, T, seed=9)
    ws = torch.empty(m.moesq_layer_host_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device="cuda")
    xh = torch.from_numpy(x.view(np.int16).copy()).pin_memory()
    lh = torch.from_numpy(lg).pin_memory()
    oh = torch.empty(T, H, dtype=torch.int16).pin_memory()
    m.moesq_moe_layer_host(xh, lh, T, k, pw_gu, pw_dn, to_dev(ga), to_dev(gh), oh, ws)
    assert (oh.numpy().view(np.uint16) == out).all()


def test_calibration_matches_oracle(cuda_lib):
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, k, H, I, T = 8, 2, 512, 256, 64
    out, ref, (x, lg, ga, gh, pw_gu, pw_dn, ws, _, _) = _layer_case(m, E, k, H, I, T, seed=13)
    g1 = torch.empty(E, dtype=torch.float32, device="cuda")
    g2 = torch.empty(E, dtype=torch.float32, device="cuda")
    m.moesq_calibrate_layer(to_dev(x), to_dev(lg), T, k, pw_gu, pw_dn, g1, g2, ws)
    assert m.moesq_get_device_error()[0] == 0
    assert (to_np(g1) == ga).all()                       # amax of bf16 inputs: exact
    assert np.allclose(to_np(g2), gh, rtol=2e-2)         # via the bf16 gate_up output
