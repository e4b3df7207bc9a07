"""GPU parity of the C-ABI entry points against the oracle, on seeded inputs.

Sizes span several blocks and a ragged tail (d_ff not a multiple of the grid, several
32-neuron words per block), plus the single-layer shapes of the full workloads."""
import numpy as np
import pytest
import torch

import pi_synth as S
from oracle import cpp as OC
from oracle import ffn as O
import gpu_helpers as H

pytestmark = pytest.mark.gpu

pi = pytest.importorskip("activation_sparse_decode_bitmask_b200")

# ----------------------------------------------------------------- small workloads
W_F32_CAL = S.FFN512_CAL
W_F32_LIT = S.FFN512_LIT
W_F16_REGLU = S.scaled(S.LLAMA2_7B, "reglu_f16_d1024", 4, 1024, 4192, 128)
W_F16_RELU = S.scaled(S.FALCON_40B, "relu_f16_d1024", 3, 1024, 4096 + 64, 128)
W_Q4_REGLU = S.scaled(S.LLAMA2_70B_Q4, "reglu_q4_d512", 3, 512, 2048 + 32, 64)
W_F32_RELU_STACK = S.FFN512_CAL.with_(name="relu_f32_stack", n_layers=3)
SMALL = [W_F32_CAL, W_F32_LIT, W_F16_REGLU, W_F16_RELU, W_Q4_REGLU]


def _ws(wl, B=4, L=None):
    return pi.Workspace(wl.d_model, wl.d_ff, wl.rank, B, L or max(1, wl.n_layers))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


# ----------------------------------------------------------------- predictor
@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_predict_parity(wl, B):
    if wl.w_dtype == "q4_0" and B > 2:
        pytest.skip("Q4_0 fused path serves batch <= 2")
    gl, sl = H.build_layers(pi, wl, 1)
    ws = _ws(wl)
    x = S.make_inputs(wl, B, "cuda", stream_id=B)
    mask = torch.full((B, wl.d_ff // 32), 0xFFFFFFFF, dtype=torch.int64).to(torch.int32).cuda()
    logits = torch.empty(B, wl.d_ff, device="cuda")
    pi.predict(gl[0], x, B, mask, logits, ws)
    assert ws.status() == 0
    lref = H.oracle_logits(sl[0], H.x_to_np(x))
    lg = logits.cpu().double().numpy()
    scale = max(1.0, float(np.max(np.abs(lref))))
    assert np.max(np.abs(lg - lref)) <= 1e-4 * scale, np.max(np.abs(lg - lref))
    bits = H.unpack_words(mask, wl.d_ff)
    assert np.array_equal(bits, lg > 0), "mask words disagree with the kernel's own logits"
    bad, flips, band = H.mask_parity(lref, bits)
    assert bad == 0, (bad, flips, band)
    print(f"{wl.name} B={B}: active/token {bits.sum(1).tolist()}, band {band}, in-band flips {flips}")


# ----------------------------------------------------------------- compaction
@pytest.mark.parametrize("B,f,dens", [(1, 64, 0.0), (1, 64, 1.0), (1, 2048, 0.1), (3, 4192, 0.05),
                                      (8, 11008, 0.1), (32, 49152, 0.1), (1, 32768 + 32, 0.5),
                                      (16, 1024 * 32, 0.002)])
def test_compact_parity(B, f, dens):
    rng = np.random.default_rng(f + B)
    bits = rng.random((B, f)) < dens
    words = O.pack_mask(bits)
    ref_idx, ref_cnt = O.compact(words, f)
    m = torch.from_numpy(words.view(np.int32)).cuda()
    idx = torch.full((f,), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    pi.compact_active(m, B, f, idx, cnt)
    torch.cuda.synchronize()
    assert int(cnt.item()) == ref_cnt
    got = idx.cpu().numpy()
    assert np.array_equal(got[:ref_cnt], ref_idx)
    assert np.all(got[ref_cnt:] == -7), "wrote past count"


# ----------------------------------------------------------------- sparse FFN
@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("B", [1, 2, 4])
def test_sparse_ffn_parity(wl, B):
    if wl.w_dtype == "q4_0" and B > 2:
        pytest.skip("Q4_0 fused path serves batch <= 2")
    gl, sl = H.build_layers(pi, wl, 1)
    ws = _ws(wl)
    x = S.make_inputs(wl, B, "cuda", stream_id=10 + B)
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
    print(f"{wl.name} B={B}: count {cnt}, y rel err {err:.2e}")


@pytest.mark.parametrize("wl", [W_F32_CAL, W_F16_REGLU, W_Q4_REGLU], ids=lambda w: w.name)
def test_sparse_equals_dense_on_gpu(wl):
    """With the true activation mask, the sparse FFN equals the dense FFN (skipped
    neurons contribute exact zeros): the GPU's sparse result matches the oracle's dense
    result within the tolerance."""
    gl, sl = H.build_layers(pi, wl, 1)
    ws = _ws(wl)
    x = S.make_inputs(wl, 1, "cuda", stream_id=21)
    xn = H.x_to_np(x)
    cl = H.cpp_layer(sl[0])
    m = cl.true_mask(xn)
    words = O.pack_mask(m)
    idx, cnt = O.compact(words, wl.d_ff)
    y_dense = cl.dense_ffn(xn)
    y = torch.empty(1, wl.d_model, device="cuda")
    pi.sparse_ffn(gl[0], x, 1, torch.from_numpy(words.view(np.int32)).cuda(),
                  torch.from_numpy(idx).cuda(), torch.tensor([cnt], dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 0
    assert H.rel_err(y.cpu().double().numpy(), y_dense) <= H.y_tol(wl.w_dtype)


def test_sparse_ffn_empty_list():
    wl = W_F16_REGLU
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    ws = _ws(wl)
    x = S.make_inputs(wl, 1, "cuda")
    y = torch.full((1, wl.d_model), 5.0, device="cuda")
    z = torch.zeros(1, wl.d_ff // 32, dtype=torch.int32, device="cuda")
    pi.sparse_ffn(gl[0], x, 1, z, torch.zeros(1, dtype=torch.int32, device="cuda"),
                  torch.zeros(1, dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 0
    assert torch.count_nonzero(y).item() == 0


def test_sparse_ffn_rejects_bad_count():
    wl = W_F16_REGLU
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    ws = _ws(wl)
    x = S.make_inputs(wl, 1, "cuda")
    y = torch.empty(1, wl.d_model, device="cuda")
    z = torch.zeros(1, wl.d_ff // 32, dtype=torch.int32, device="cuda")
    idx = torch.zeros(wl.d_ff, dtype=torch.int32, device="cuda")
    pi.sparse_ffn(gl[0], x, 1, z, idx, torch.tensor([wl.d_ff + 1], dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 6          # PI_ERR_DEVICE, reported, not a fault
    # the workspace stays usable
    pi.sparse_ffn(gl[0], x, 1, z, idx, torch.zeros(1, dtype=torch.int32, device="cuda"), y, ws)
    assert ws.status() == 0


# ----------------------------------------------------------------- decode stack
def _stack_check(wl, B, n_layers, stream_id=0):
    """Run the stack on the GPU from x0 and compare layer by layer with the oracle's own
    trajectory.  When a mask bit flips inside the band (both results are correct), the
    GPU's segment from that layer on is re-run from the oracle's next input."""
    gl, sl = H.build_layers(pi, wl, n_layers)
    cls = [H.cpp_layer(L) for L in sl]
    ws = _ws(wl, B=B, L=n_layers)
    xdt = torch.float32 if wl.x_dtype == "f32" else torch.float16
    x0 = S.make_inputs(wl, B, "cuda", stream_id=stream_id)
    ref = OC.decode_stack(H.x_to_np(x0), cls, wl.x_dtype)
    total_flips, l0, x_start, resyncs = 0, 0, x0, 0
    tol = H.y_tol(wl.w_dtype)
    words = wl.d_ff // 32
    while l0 < n_layers:
        n = n_layers - l0
        tr = {"x": torch.empty(n + 1, B, wl.d_model, device="cuda", dtype=xdt),
              "logits": torch.empty(n, B, wl.d_ff, device="cuda"),
              "mask": torch.empty(n, B, words, device="cuda", dtype=torch.int32),
              "idx": torch.empty(n, wl.d_ff, device="cuda", dtype=torch.int32),
              "count": torch.empty(n, device="cuda", dtype=torch.int32),
              "y": torch.empty(n, B, wl.d_model, device="cuda")}
        xio = x_start.clone()
        pi.decode_stack(gl[l0:], xio, B, ws, trace=tr)
        assert ws.status() == 0
        assert torch.equal(tr["x"][n], xio), "returned x differs from the trace's last entry"
        flipped_at = None
        for k in range(n):
            l = l0 + k
            r = ref[l]
            lg = tr["logits"][k].cpu().double().numpy()
            bits = H.unpack_words(tr["mask"][k], wl.d_ff)
            assert np.array_equal(bits, lg > 0)
            idx_ref, cnt_ref = O.compact(O.pack_mask(bits), wl.d_ff)
            cnt = int(tr["count"][k].item())
            assert cnt == cnt_ref and np.array_equal(tr["idx"][k, :cnt].cpu().numpy(), idx_ref)
            bad, flips, _ = H.mask_parity(r["logits"], bits)
            assert bad == 0, f"layer {l}: {bad} mask bits differ outside the band"
            xg = tr["x"][k].cpu().double().numpy()
            assert np.max(np.abs(xg - r["x_in"])) <= 2.0 ** -9 * (1 + np.max(np.abs(r["x_in"]))), \
                f"layer {l} input drifted"
            y = tr["y"][k].cpu().double().numpy()
            if flips:
                # the GPU took the other (equally valid) side of a band neuron: its y must
                # be the oracle's y on the oracle mask with those band bits set the GPU's
                # way (outside the band the two masks were checked equal above)
                in_band = np.abs(r["logits"]) < H.BAND
                alt = np.where(in_band, bits, r["logits"] > 0)
                alt_idx, _ = O.compact(O.pack_mask(alt), wl.d_ff)
                y_alt = cls[l].sparse_ffn(r["x_in"], alt, alt_idx)
                assert H.rel_err(y, y_alt) <= tol
                total_flips += flips
                flipped_at = l
                break
            assert H.rel_err(y, r["y"]) <= tol, f"layer {l}: y rel err {H.rel_err(y, r['y'])}"
        if flipped_at is None:
            xf = xio.cpu().double().numpy()
            assert np.max(np.abs(xf - ref[-1]["x_next"])) <= 2.0 ** -9 * (1 + np.max(np.abs(ref[-1]["x_next"])))
            break
        l0 = flipped_at + 1
        if l0 < n_layers:
            x_start = torch.from_numpy(np.asarray(ref[l0]["x_in"])).to(device="cuda", dtype=xdt)
            resyncs += 1
    return total_flips, resyncs


@pytest.mark.parametrize("wl,B", [(W_F32_RELU_STACK, 1), (W_F16_REGLU, 1), (W_F16_REGLU, 2), (W_F16_RELU, 1),
                                  (W_F16_RELU, 4), (W_Q4_REGLU, 1), (W_Q4_REGLU, 2)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_decode_stack_parity(wl, B):
    flips, resyncs = _stack_check(wl, B, wl.n_layers, stream_id=30 + B)
    print(f"{wl.name} B={B}: in-band flips {flips}, re-syncs {resyncs}")


def test_decode_stack_deterministic():
    wl = W_F16_REGLU
    gl, _ = H.build_layers(pi, wl, keep_host=False)
    ws = _ws(wl, B=1)
    x0 = S.make_inputs(wl, 1, "cuda", stream_id=3)
    outs = []
    for _ in range(3):
        x = x0.clone()
        pi.decode_stack(gl, x, 1, ws)
        outs.append(x)
    assert ws.status() == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_decode_stack_host_matches_device():
    wl = W_F16_RELU
    gl, _ = H.build_layers(pi, wl, keep_host=False)
    ws = _ws(wl, B=2)
    x0 = S.make_inputs(wl, 2, "cuda", stream_id=4)
    xd = x0.clone()
    pi.decode_stack(gl, xd, 2, ws)
    assert ws.status() == 0
    xh = x0.cpu().pin_memory()
    out = torch.empty_like(xh).pin_memory()
    pi.decode_stack_host(gl, xh, out, 2, ws)
    assert torch.equal(out, xd.cpu())


# ----------------------------------------------------------------- hot reorder
@pytest.mark.parametrize("wl", [W_F16_REGLU, W_Q4_REGLU, W_F32_CAL], ids=lambda w: w.name)
def test_reorder_hot_prefix(wl):
    gl, sl = H.build_layers(pi, wl, 1)
    ws = _ws(wl)
    L = sl[0]
    freq = L.freq.clone()
    freq[::7] = freq[3]          # ties must break by original index
    pi.reorder_hot_prefix(gl[0], freq)
    perm = torch.empty(wl.d_ff, dtype=torch.int32, device="cuda")
    pi.get_perm(gl[0], perm)
    perm = perm.cpu().numpy()
    assert np.array_equal(perm, O.hot_order(freq.cpu().numpy()))
    # the predictor's set of active original ids is unchanged, y unchanged up to order
    x = S.make_inputs(wl, 1, "cuda", stream_id=5)
    mask = torch.empty(1, wl.d_ff // 32, dtype=torch.int32, device="cuda")
    logits = torch.empty(1, wl.d_ff, device="cuda")
    pi.predict(gl[0], x, 1, mask, logits, ws)
    lref = H.oracle_logits(L, H.x_to_np(x))
    lg = logits.cpu().double().numpy()
    assert np.max(np.abs(lg[:, :] - lref[:, perm])) <= 1e-4 * max(1.0, np.max(np.abs(lref)))
    bits = H.unpack_words(mask, wl.d_ff)
    idx = torch.empty(wl.d_ff, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, dtype=torch.int32, device="cuda")
    pi.compact_active(mask, 1, wl.d_ff, idx, cnt)
    y = torch.empty(1, wl.d_model, device="cuda")
    pi.sparse_ffn(gl[0], x, 1, mask, idx, cnt, y, ws)
    assert ws.status() == 0
    c = int(cnt.item())
    orig_ids = np.sort(perm[idx[:c].cpu().numpy()])
    orig_bits = np.zeros((1, wl.d_ff), bool)
    orig_bits[0, orig_ids] = True
    y_ref = H.oracle_ffn_rows(H.x_to_np(x), L, orig_bits, orig_ids)
    assert H.rel_err(y.cpu().double().numpy(), y_ref) <= H.y_tol(wl.w_dtype)
    assert np.array_equal(bits[0, :], np.isin(np.arange(wl.d_ff), idx[:c].cpu().numpy()))


def test_reorder_rejects_nan():
    wl = W_F16_RELU
    gl, sl = H.build_layers(pi, wl, 1)
    freq = sl[0].freq.clone()
    freq[5] = float("nan")
    with pytest.raises(pi.PiError):
        pi.reorder_hot_prefix(gl[0], freq)


# ----------------------------------------------------------------- failure reporting
def test_barrier_timeout_is_reported_not_hung():
    """A grid-barrier wait that can never complete gives up after its limit, the error
    word says so, and the workspace is usable afterwards."""
    wl = W_F16_REGLU
    ws = _ws(wl)
    pi.diag_barrier_timeout(ws, 20_000_000)           # 20 ms
    assert ws.status() == 5                           # PI_ERR_TIMEOUT
    gl, _ = H.build_layers(pi, wl, 2, keep_host=False)
    x = S.make_inputs(wl, 1, "cuda")
    pi.decode_stack(gl, x, 1, ws)
    assert ws.status() == 0


def test_argument_errors():
    wl = W_F16_REGLU
    ws = _ws(wl)
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    x = S.make_inputs(wl, 1, "cuda")
    mask = torch.empty(40, wl.d_ff // 32, dtype=torch.int32, device="cuda")
    with pytest.raises(pi.PiError) as e:
        pi.predict(gl[0], x, 0, mask, None, ws)
    assert e.value.status == 1
    with pytest.raises(pi.PiError):
        pi.predict(gl[0], x, 33, mask, None, ws)
    small = pi.Workspace(256, 1024, 64, 1, 1)
    with pytest.raises(pi.PiError):
        pi.predict(gl[0], x, 1, mask, None, small)


def test_allocation_failure_is_reported():
    """A workspace larger than the device can hold returns PI_ERR_OOM from the allocation
    (no fault, nothing left allocated), and the device goes on working."""
    free0, _ = torch.cuda.mem_get_info()
    with pytest.raises(pi.PiError) as e:
        pi.Workspace(4096, 1 << 30, 512, pi.PI_MAX_BATCH, 1)   # h words alone: 2^30 x 32 x 8 bytes
    assert e.value.status == 3                                # PI_ERR_OOM
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert abs(free1 - free0) < (64 << 20), (free0, free1)
    wl = W_F16_REGLU
    gl, _ = H.build_layers(pi, wl, 1, keep_host=False)
    ws = _ws(wl)
    x = S.make_inputs(wl, 1, "cuda")
    pi.decode_stack(gl, x, 1, ws)
    assert ws.status() == 0


# ----------------------------------------------------------------- per-layer predictor rank
W_MIXED_RANK = S.scaled(S.LLAMA2_7B, "reglu_f16_mixed_rank", 3, 1024, 4192, 384, layer_rank=(256, 128, 384))


@pytest.mark.parametrize("B", [1, 2, 8])
def test_decode_stack_mixed_rank(B):
    """Layers of one stack with different predictor ranks (unite.ai "PowerInfer: Mesin
    Inferensi LLM Cepat dengan GPU Konsumen", §"Prediktor Kepadatan Adaptif": each layer's
    predictor is sized on its own) run in one call and match the oracle layer by layer."""
    assert [W_MIXED_RANK.at_layer(l).rank for l in range(3)] == [256, 128, 384]
    flips, resyncs = _stack_check(W_MIXED_RANK, B, 3, stream_id=600 + B)
    print(f"mixed-rank stack B={B}: in-band flips {flips}, re-syncs {resyncs}")


def test_decode_stack_rejects_other_shapes():
    """Only the rank may differ between the layers of a stack."""
    a = S.scaled(S.LLAMA2_7B, "reglu_f16_d1024_a", 1, 1024, 4192, 128)
    b = S.scaled(S.LLAMA2_7B, "reglu_f16_d1024_b", 1, 1024, 4096, 128)
    ga, _ = H.build_layers(pi, a, 1, keep_host=False)
    gb, _ = H.build_layers(pi, b, 1, keep_host=False)
    ws = _ws(a, B=1, L=2)
    x = S.make_inputs(a, 1, "cuda")
    with pytest.raises(pi.PiError) as e:
        pi.decode_stack([ga[0], gb[0]], x, 1, ws)
    assert e.value.status == 1


# ----------------------------------------------------------------- row-owned down pass
# d = 1024 keeps a down-list chunk at its 1024-entry cap; ~4900 active neurons a layer
# (15 % of 32768) exceed three chunks, so one token takes the row-owned down pass.
W_ROW_OWNED = [S.scaled(S.FALCON_40B, "relu_f16_row_owned", 2, 1024, 32768, 128, mean_p=0.15),
               S.scaled(S.LLAMA2_70B_Q4, "reglu_q4_row_owned", 2, 1024, 32768, 128, mean_p=0.15)]


@pytest.mark.parametrize("wl", W_ROW_OWNED, ids=lambda w: w.name)
def test_decode_stack_row_owned_down(wl):
    """A stack whose layers are past three down-list chunks (each block sums the full down
    rows of the records it dots and the blocks exchange partial y) matches the oracle
    layer by layer, as the column-owned pass does (the down projection is the same sum,
    KPD "PowerInfer: Fast Large Language Model Serving with a Consumer-grade GPU",
    §"Метод": only the active neurons' rows and columns are read)."""
    flips, resyncs = _stack_check(wl, 1, wl.n_layers, stream_id=700)
    print(f"{wl.name}: in-band flips {flips}, re-syncs {resyncs}")
