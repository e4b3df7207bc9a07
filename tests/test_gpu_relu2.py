"""GPU parity of the squared-ReLU family (a_i = max(0, w_up_i . x + b_i)^2, the third
activation family the pages list as supported: GeekNews "Tüketici sınıfı GPU takılı
PC'lerde yüksek hızlı büyük dil modeli serving", §"Kısıtlar ve SSS") against the
oracle, through the C ABI: the single-launch path at 1 to 4 tokens, the multi-launch
path at 5 to 32 tokens, and a decode stack."""
import numpy as np
import pytest
import torch

import pi_synth as S
from oracle import ffn as O
import gpu_helpers as H
from test_gpu_parity import _stack_check

pytestmark = pytest.mark.gpu
pi = pytest.importorskip("activation_sparse_decode_bitmask_b200")

W_F16 = S.scaled(S.FALCON_40B, "relu2_f16_d1024", 3, 1024, 4096 + 64, 128, act="relu2")
W_F32 = S.FFN512_CAL.with_(name="relu2_f32", act="relu2", n_layers=2)
W_Q4 = S.scaled(S.LLAMA2_70B_Q4, "relu2_q4_d512", 2, 512, 2048 + 32, 64, act="relu2")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def test_relu2_enum_in_abi():
    assert pi.PI_RELU2 == 2
    d = pi.make_desc(512, 2048, 64, "relu2", "f16", "f16", "f16")
    assert d.act == pi.PI_RELU2


@pytest.mark.parametrize("wl,B", [(W_F16, 1), (W_F16, 2), (W_F16, 4), (W_F32, 1), (W_F32, 3), (W_Q4, 1), (W_Q4, 2),
                                  (W_F16, 5), (W_F16, 8), (W_F16, 32)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_relu2_sparse_ffn_parity(wl, B):
    gl, sl = H.build_layers(pi, wl, 1)
    ws = pi.Workspace(wl.d_model, wl.d_ff, wl.rank, max(B, 4), 1)
    x = S.make_inputs(wl, B, "cuda", stream_id=400 + B)
    xn = H.x_to_np(x)
    bits = O.fire_bits(H.oracle_logits(sl[0], xn))
    words = O.pack_mask(bits)
    idx, cnt = O.compact(words, wl.d_ff)
    y_ref = H.oracle_ffn_rows(xn, sl[0], bits, idx)
    y = torch.full((B, wl.d_model), float("nan"), device="cuda")
    pi.sparse_ffn(gl[0], x, B, torch.from_numpy(words.view(np.int32)).cuda(),
                  torch.from_numpy(np.concatenate([idx, np.zeros(1, np.int32)])).cuda(),
                  torch.tensor([cnt], dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 0
    err = H.rel_err(y.cpu().double().numpy(), y_ref)
    assert err <= H.y_tol(wl.w_dtype), err
    # the square is applied: the same rows under ReLU give a different output
    relu = H.cpp_layer_as(sl[0], "relu").sparse_ffn(xn, bits, idx)
    assert H.rel_err(relu, y_ref) > 10 * H.y_tol(wl.w_dtype)
    print(f"{wl.name} B={B}: count {cnt}, y rel err {err:.2e}")


@pytest.mark.parametrize("wl,B", [(W_F16, 1), (W_F16, 2), (W_Q4, 1), (W_F16, 8)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_relu2_decode_stack_parity(wl, B):
    flips, resyncs = _stack_check(wl, B, wl.n_layers, stream_id=450 + B)
    print(f"{wl.name} B={B}: in-band flips {flips}, re-syncs {resyncs}")
