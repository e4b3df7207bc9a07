"""pi_predict_noalloc: the predictor launch of pi_predict with its cross-block scratch in
one static device array instead of a workspace.  Checked through the C ABI against
pi_predict on the same layer and inputs (the same bits and the same logits, since both
run the same launch), and against the oracle, on two calls in a row.

The file name puts it last in collection order, so that it runs both on its own and
after every other GPU test has used workspaces on the same device."""
import numpy as np
import pytest
import torch

import pi_synth as S
import gpu_helpers as H

pytestmark = pytest.mark.gpu
pi = pytest.importorskip("activation_sparse_decode_bitmask_b200")

W_F16_REGLU = S.scaled(S.LLAMA2_7B, "reglu_f16_d1024", 1, 1024, 4192, 128)
W_F16_RELU = S.scaled(S.FALCON_40B, "relu_f16_d1024", 1, 1024, 4096 + 64, 128)
W_Q4_REGLU = S.scaled(S.LLAMA2_70B_Q4, "reglu_q4_d512", 1, 512, 2048 + 32, 64)
W_WIDE_RANK = S.scaled(S.LLAMA2_7B, "reglu_f16_d1024_r1024", 1, 1024, 4192, 1024)
CASES = [(S.FFN512_CAL, 3), (W_F16_REGLU, 1), (W_F16_REGLU, 4), (W_F16_RELU, 2), (W_Q4_REGLU, 2),
         (S.LLAMA2_7B, 1)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _reference(layer, wl, B, x):
    ws = pi.Workspace(wl.d_model, wl.d_ff, wl.rank, B, 1)
    mask = torch.empty(B, wl.d_ff // 32, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, wl.d_ff, device="cuda")
    pi.predict(layer, x, B, mask, logits, ws)
    assert ws.status() == 0
    return mask, logits


def _noalloc(layer, wl, B, x):
    mask = torch.full((B, wl.d_ff // 32), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    logits = torch.full((B, wl.d_ff), float("nan"), device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    pi.predict_noalloc(layer, x, B, mask, logits, status)
    torch.cuda.synchronize()
    return mask, logits, int(status.item())


def _agree(wl, mask, logits, mask_ref, logits_ref, lref=None):
    """Bit-for-bit equal to pi_predict's outputs; within the parity bars of the oracle's
    logits where those are given."""
    assert torch.equal(mask, mask_ref), "mask words differ from pi_predict's"
    assert torch.equal(logits, logits_ref), "logits differ from pi_predict's"
    lg = logits.double().cpu().numpy()
    bits = H.unpack_words(mask, wl.d_ff)
    assert np.array_equal(bits, lg > 0), "mask words disagree with the call's own logits"
    if lref is not None:
        scale = max(1.0, float(np.max(np.abs(lref))))
        assert np.max(np.abs(lg - lref)) <= 1e-4 * scale, np.max(np.abs(lg - lref))
        bad, _, _ = H.mask_parity(lref, bits)
        assert bad == 0


@pytest.mark.parametrize("wl,B", CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_noalloc_matches_predict(wl, B):
    gl, sl = H.build_layers(pi, wl, 1)
    x = S.make_inputs(wl, B, "cuda", stream_id=31 + B)
    mask_ref, logits_ref = _reference(gl[0], wl, B, x)
    lref = H.oracle_logits(sl[0], H.x_to_np(x))
    for call in range(2):   # the second call starts from the scratch the first one left
        mask, logits, st = _noalloc(gl[0], wl, B, x)
        assert st == 0, (call, pi.status_str(st))
        _agree(wl, mask, logits, mask_ref, logits_ref, lref)


def test_noalloc_interleaved_batches():
    """Calls of different batch sizes, with workspace calls between them, on one layer:
    words an earlier call left in the scratch never stand in for a later call's."""
    wl = W_F16_REGLU
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    for B in (4, 1, 2, 4, 1):
        x = S.make_inputs(wl, B, "cuda", stream_id=50 + B)
        mask, logits, st = _noalloc(gl[0], wl, B, x)
        assert st == 0
        mask_ref, logits_ref = _reference(gl[0], wl, B, x)
        _agree(wl, mask, logits, mask_ref, logits_ref)


def test_noalloc_allocates_nothing():
    wl = W_F16_REGLU
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    B = 2
    x = S.make_inputs(wl, B, "cuda", stream_id=60)
    mask = torch.empty(B, wl.d_ff // 32, dtype=torch.int32, device="cuda")
    logits = torch.empty(B, wl.d_ff, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pi.predict_noalloc(gl[0], x, B, mask, logits, status)   # set-up and module loads happen here
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        pi.predict_noalloc(gl[0], x, B, mask, logits, status)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert int(status.item()) == 0
    assert free1 == free0, (free0, free1)


def test_noalloc_rejects_oversized_scratch():
    """A shape whose scratch exceeds PI_NOALLOC_SCRATCH_BYTES is refused before anything
    is enqueued; a valid call afterwards still works."""
    wl = W_WIDE_RANK   # 32 tokens x rank 1024 of tagged u words alone fill the array
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    B = pi.PI_MAX_BATCH
    need = 256 + -(-(B * wl.rank * 8) // 256) * 256
    assert need > pi.PI_NOALLOC_SCRATCH_BYTES
    x = S.make_inputs(wl, B, "cuda", stream_id=70)
    mask = torch.full((B, wl.d_ff // 32), 7, dtype=torch.int32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    with pytest.raises(pi.PiError) as e:
        pi.predict_noalloc(gl[0], x, B, mask, None, status)
    assert e.value.status == 2   # PI_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(status.item()) == -1 and bool((mask == 7).all())
    with pytest.raises(pi.PiError) as e:   # the status word is required
        pi.predict_noalloc(gl[0], x[:1], 1, mask[:1], None, None)
    assert e.value.status == 1
    m, lg, st = _noalloc(gl[0], wl, 1, x[:1].contiguous())
    assert st == 0
    mask_ref, logits_ref = _reference(gl[0], wl, 1, x[:1].contiguous())
    _agree(wl, m, lg, mask_ref, logits_ref)


@pytest.mark.parametrize("wl,B", [(W_F16_REGLU, 5), (S.scaled(S.FALCON_40B, "relu_f16_d8192", 1, 8192, 2048, 128), 4),
                                  (W_Q4_REGLU, 3)],
                         ids=["5 tokens", "d 8192 at 4 tokens", "Q4_0 at 3 tokens"])
def test_noalloc_unsupported_shape_enqueues_nothing(wl, B):
    """Shapes only pi_predict's multi-launch path serves are refused before anything is
    enqueued: the mask and the status word keep their contents and no kernel starts."""
    lay = _zero_layer(wl)
    x = torch.zeros(B, wl.d_model, dtype=torch.float16, device="cuda")
    mask = torch.full((B, wl.d_ff // 32), 7, dtype=torch.int32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    n0 = pi.kernel_launches()
    with pytest.raises(pi.PiError) as e:
        pi.predict_noalloc(lay, x, B, mask, None, status)
    assert e.value.status == 2   # PI_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert pi.kernel_launches() == n0
    assert int(status.item()) == -1 and bool((mask == 7).all())


def _zero_layer(wl):
    """A layer of the workload's shape with zero weights (only the shape matters here)."""
    d, f, r = wl.d_model, wl.d_ff, wl.rank
    t = {"bias": torch.zeros(f, device="cuda"), "thresh": torch.zeros(f, device="cuda"),
         "p1": torch.zeros(d, r, dtype=torch.float16, device="cuda"),
         "p2": torch.zeros(r, f, dtype=torch.float16, device="cuda")}
    if wl.w_dtype == "q4_0":
        for m in ("up", "down") + (("gate",) if wl.act == "reglu" else ()):
            t["q_" + m] = torch.zeros(f, d // 32, 16, dtype=torch.uint8, device="cuda")
            t["s_" + m] = torch.zeros(f, d // 32, dtype=torch.float16, device="cuda")
    else:
        t["w_up"] = torch.zeros(f, d, dtype=torch.float16, device="cuda")
        t["w_down"] = torch.zeros(d, f, dtype=torch.float16, device="cuda")
        if wl.act == "reglu":
            t["w_gate"] = torch.zeros(f, d, dtype=torch.float16, device="cuda")
    return pi.load_layer(H.desc_of(pi, wl), t)
