"""GPU parity of the batched path (5 to 32 tokens per call, fp16 family: tensor-core tiles
for the predictor, the gate/up rows and the down columns of the active neurons) against
the oracle, through the C ABI.  Same bars as the batch-1 path: mask bits exact outside
the 1e-3 band of the fp64 logits, FFN output within 1e-2 * max|y_ref|."""
import numpy as np
import pytest
import torch

import pi_synth as S
from oracle import ffn as O
import gpu_helpers as H
from test_gpu_parity import _stack_check

pytestmark = pytest.mark.gpu
pi = pytest.importorskip("activation_sparse_decode_bitmask_b200")

W_OPT_SMALL = S.scaled(S.OPT_175B, "relu_f16_opt_d1024", 3, 1024, 4096 + 64, 128)
W_REGLU_SMALL = S.scaled(S.LLAMA2_7B, "reglu_f16_d1024", 3, 1024, 4192, 128)
SMALL = [W_OPT_SMALL, W_REGLU_SMALL]
BATCHES = [5, 8, 16, 32]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _ws(wl, B, L=1):
    return pi.Workspace(wl.d_model, wl.d_ff, wl.rank, B, L)


def _predict_check(gl, L, wl, B, ws, stream_id):
    x = S.make_inputs(wl, B, "cuda", stream_id=stream_id)
    mask = torch.full((B, wl.d_ff // 32), -1, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, wl.d_ff, device="cuda")
    pi.predict(gl, x, B, mask, logits, ws)
    assert ws.status() == 0
    lref = H.oracle_logits(L, H.x_to_np(x))
    lg = logits.cpu().double().numpy()
    scale = max(1.0, float(np.max(np.abs(lref))))
    assert np.max(np.abs(lg - lref)) <= 1e-4 * scale, np.max(np.abs(lg - lref))
    bits = H.unpack_words(mask, wl.d_ff)
    assert np.array_equal(bits, lg > 0), "mask words disagree with the kernel's own logits"
    bad, flips, band = H.mask_parity(lref, bits)
    assert bad == 0, (bad, flips, band)
    return x, lref, bits, flips


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("B", BATCHES)
def test_batched_predict_parity(wl, B):
    gl, sl = H.build_layers(pi, wl, 1)
    _, _, bits, flips = _predict_check(gl[0], sl[0], wl, B, _ws(wl, B), 100 + B)
    print(f"{wl.name} B={B}: union active {int(bits.any(0).sum())}/{wl.d_ff}, in-band flips {flips}")


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("B", BATCHES)
def test_batched_ffn_parity(wl, B):
    gl, sl = H.build_layers(pi, wl, 1)
    ws = _ws(wl, B)
    x = S.make_inputs(wl, B, "cuda", stream_id=120 + B)
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
    print(f"{wl.name} B={B}: union count {cnt}, y rel err {err:.2e}")


def test_batched_ffn_empty_and_bad_count():
    wl = W_REGLU_SMALL
    B = 8
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    ws = _ws(wl, B)
    x = S.make_inputs(wl, B, "cuda")
    z = torch.zeros(B, wl.d_ff // 32, dtype=torch.int32, device="cuda")
    idx = torch.zeros(wl.d_ff, dtype=torch.int32, device="cuda")
    y = torch.full((B, wl.d_model), 5.0, device="cuda")
    pi.sparse_ffn(gl[0], x, B, z, idx, torch.zeros(1, dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 0
    assert torch.count_nonzero(y).item() == 0          # empty list: y = 0
    pi.sparse_ffn(gl[0], x, B, z, idx, torch.tensor([wl.d_ff + 1], dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 6                            # PI_ERR_DEVICE, reported, not a fault
    bad_idx = torch.full((wl.d_ff,), wl.d_ff + 5, dtype=torch.int32, device="cuda")
    pi.sparse_ffn(gl[0], x, B, z, bad_idx, torch.tensor([3], dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 6
    pi.sparse_ffn(gl[0], x, B, z, idx, torch.zeros(1, dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 0                            # the workspace stays usable


@pytest.mark.parametrize("wl,B", [(W_OPT_SMALL, 8), (W_OPT_SMALL, 32), (W_REGLU_SMALL, 16)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_batched_stack_parity(wl, B):
    flips, resyncs = _stack_check(wl, B, wl.n_layers, stream_id=140 + B)
    print(f"{wl.name} B={B}: in-band flips {flips}, re-syncs {resyncs}")


def test_batched_stack_deterministic():
    wl = W_OPT_SMALL
    B = 16
    gl, _ = H.build_layers(pi, wl, keep_host=False)
    ws = _ws(wl, B, wl.n_layers)
    x0 = S.make_inputs(wl, B, "cuda", stream_id=160)
    outs = []
    for _ in range(2):
        x = x0.clone()
        pi.decode_stack(gl, x, B, ws)
        assert ws.status() == 0
        outs.append(x)
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("B", [8, 32])
def test_batched_fullsize_opt_layer(B):
    """One OPT-175B-shaped layer (d 12288, d_ff 49152, rank 1536) at 8 and 32 tokens: the
    predictor against the fp64 oracle, and the FFN on the oracle's own mask."""
    wl = S.OPT_175B
    gl, sl = H.build_layers(pi, wl, 1)
    ws = _ws(wl, B)
    x, lref, _, flips = _predict_check(gl[0], sl[0], wl, B, ws, 180 + B)
    xn = H.x_to_np(x)
    rb = O.fire_bits(lref)
    words = O.pack_mask(rb)
    idx, cnt = O.compact(words, wl.d_ff)
    y = torch.empty(B, wl.d_model, device="cuda")
    pi.sparse_ffn(gl[0], x, B, torch.from_numpy(words.view(np.int32)).cuda(), torch.from_numpy(idx).cuda(),
                  torch.tensor([cnt], dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 0
    y_ref = H.oracle_ffn_rows(xn, sl[0], rb, idx)
    err = H.rel_err(y.cpu().double().numpy(), y_ref)
    assert err <= H.y_tol(wl.w_dtype), err
    print(f"OPT-175B layer B={B}: union {cnt}/{wl.d_ff}, in-band flips {flips}, y rel err {err:.2e}")


def test_kernel_launch_count_per_step():
    """pi_kernel_launches brackets the launches of a call: one persistent launch per decode
    step at one token, eleven launches per layer on the batched path (predictor rows and
    epilogue twice, compaction, count, gate/up rows and epilogue, down, down reduce, glue)."""
    wl = W_OPT_SMALL
    gl, _ = H.build_layers(pi, wl, keep_host=False)
    L = wl.n_layers
    for B, per_step in [(1, 1), (8, 11 * L)]:
        ws = _ws(wl, B, L)
        x = S.make_inputs(wl, B, "cuda", stream_id=170 + B)
        n0 = pi.kernel_launches()
        pi.decode_stack(gl, x, B, ws)
        n1 = pi.kernel_launches()
        assert ws.status() == 0
        assert n1 - n0 == per_step, (B, n1 - n0)
