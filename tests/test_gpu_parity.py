"""GPU parity of every step of the hot path against the CPU oracle.

All calls go through the C ABI (libsparge.so via the ctypes binding).  Masks
and index work must match bit-exactly (mask entries the oracle marks as
ambiguous excepted); float outputs must meet the stated tolerances on the
float32 output mode, and 16-bit outputs must be within one ulp of the oracle
rounded to the same dtype."""
import numpy as np
import pytest
import torch

import free_block_sparse_predict_b200 as fb
from oracle import sparge_oracle as orc
from synth import bf16_bits_from_f32, to_f32, to_f64

from gpu_common import (INT8_COS, INT8_REL_L1, MAX_ABS, MEAN_REL_L1, check_mask,
                        compare_rows, dev, gpu_attention, gpu_compact, gpu_predict,
                        oracle_inputs, params_for, report_lambda, sample_tiles, tile_rows,
                        to_dev, torch_dense_attention, workload, ws_regions)

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------
# permutation
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N,P,grid", [(4608, 512, (1, 64, 64)), (17776, 226, (13, 30, 45)),
                                      (50, 3, (2, 3, 7)), (9, 0, (1, 1, 9)), (20, 4, (1, 1, 1))])
def test_hilbert_table_matches_oracle(N, P, grid):
    T, H, W = grid
    perm = torch.full((N,), -7, dtype=torch.int32, device=dev())
    ws = torch.zeros(fb.sparge_hilbert_workspace_bytes(T, H, W), dtype=torch.uint8,
                     device=dev())
    fb.sparge_hilbert_index(N, P, T, H, W, perm, ws)
    assert np.array_equal(perm.cpu().numpy(), orc.hilbert_permutation(N, P, T, H, W))


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float16, 64),
                                     (torch.float32, 64)])
def test_permute_gathers_and_inverts_exactly(dtype, d):
    N = 17776
    perm_np = orc.hilbert_permutation(N, 226, 13, 30, 45)
    perm = torch.from_numpy(perm_np.astype(np.int32)).to(dev())
    x = torch.randn(2, 3, N, d, device=dev()).to(dtype)
    y, z = torch.empty_like(x), torch.empty_like(x)
    fb.sparge_hilbert_permute(x, y, perm)
    fb.sparge_inverse_permute(y, z, perm)
    assert torch.equal(y, x[:, :, torch.from_numpy(perm_np).to(dev())])
    assert torch.equal(z, x)


@pytest.mark.parametrize("dtype,d,N,BH", [(torch.float32, 12, 1000, (1, 1)),
                                          (torch.bfloat16, 24, 333, (2, 5)),
                                          (torch.float16, 8, 1, (1, 3)),
                                          (torch.float32, 4, 70000, (1, 2))])
def test_permute_odd_rows_and_ragged_lengths(dtype, d, N, BH):
    """Rows of 3, 3, 1 and 1 vectors of 16 bytes, lengths that end inside a
    CTA's chunk: every row lands where the table says, bit for bit."""
    g = torch.Generator().manual_seed(N)
    perm_np = torch.randperm(N, generator=g).numpy().astype(np.int32)
    perm = torch.from_numpy(perm_np).to(dev())
    x = torch.randn(*BH, N, d, device=dev()).to(dtype)
    y, z = torch.empty_like(x), torch.empty_like(x)
    fb.sparge_hilbert_permute(x, y, perm)
    fb.sparge_inverse_permute(y, z, perm)
    assert torch.equal(y, x[:, :, perm.long()])
    assert torch.equal(z, x)


def test_permute_skips_table_entries_outside_the_sequence():
    N, d = 600, 64
    perm_np = np.arange(N, dtype=np.int32)[::-1].copy()
    perm_np[::7] = -1                     # rows whose entry is out of range
    perm_np[3::11] = N + 5
    perm = torch.from_numpy(perm_np).to(dev())
    x = torch.randn(1, 2, N, d, device=dev()).to(torch.bfloat16)
    y = torch.full_like(x, 7.0)
    fb.sparge_hilbert_permute(x, y, perm)
    ok = (perm_np >= 0) & (perm_np < N)
    rows = np.nonzero(ok)[0]
    assert torch.equal(y[:, :, rows], x[:, :, torch.from_numpy(perm_np[rows]).long().to(dev())])
    assert bool((y[:, :, np.nonzero(~ok)[0]] == 7.0).all())
    z = torch.full_like(x, -3.0)
    fb.sparge_inverse_permute(x, z, perm)
    tgt = torch.from_numpy(perm_np[rows]).long().to(dev())
    assert torch.equal(z[:, :, tgt], x[:, :, rows])
    untouched = np.setdiff1d(np.arange(N), perm_np[rows])
    assert bool((z[:, :, untouched] == -3.0).all())


# ----------------------------------------------------------------------------
# stage 1: predictor
# ----------------------------------------------------------------------------

PREDICT_CASES = [("tiny", {}), ("image_dit", {}), ("video_dit", {}), ("llm_32k", {})]


@pytest.mark.parametrize("name,over", PREDICT_CASES, ids=[c[0] for c in PREDICT_CASES])
def test_predict_mask_matches_oracle(name, over):
    w, t = workload(name, **over)
    Q, K, _ = oracle_inputs(w, t)
    perm = None
    if w.grid:
        perm = orc.hilbert_permutation(w.N, w.prefix_len, *w.grid)
        Q, K = orc.permute_tokens(Q, perm), orc.permute_tokens(K, perm)
    p = params_for(w)
    q = to_dev(t["q"], w.dtype)
    k = to_dev(t["k"], w.dtype)
    if perm is not None:
        pt = torch.from_numpy(perm.astype(np.int32)).to(dev())
        qp, kp = torch.empty_like(q), torch.empty_like(k)
        fb.sparge_hilbert_permute(q, qp, pt)
        fb.sparge_hilbert_permute(k, kp, pt)
        q, k = qp, kp
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, q, k)
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    check_mask(M, pr, name)
    assert np.abs(sq.cpu().numpy() - pr["s_q"]).max() < 1e-5
    assert np.abs(sk.cpu().numpy() - pr["s_k"]).max() < 1e-5
    check_pooled_means(ws, p, pr)
    # the skip list is the ascending compaction of the GPU mask
    io, co = orc.mask_compact(M)
    c = cnt.cpu().numpy()
    ii = idx.cpu().numpy()
    assert np.array_equal(c, co)
    for pos in np.ndindex(*c.shape):
        assert np.array_equal(ii[pos][:c[pos]], io[pos][:c[pos]])
    # causal-future blocks never kept
    assert not (M & ~pr["visible"]).any()


def test_predict_mask_llm_128k_full():
    w, t = workload("llm_128k")
    Q, K, _ = oracle_inputs(w, t)
    p = params_for(w)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype))
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    check_mask(M, pr, "llm_128k")
    assert np.array_equal(cnt.cpu().numpy(), M.sum(-1))


@pytest.mark.parametrize("name", ["tiny", "llm_128k"])
def test_predict_pool_then_select_equals_predict_mask(name):
    # the two halves, called apart on one workspace, give the whole call's
    # outputs bit for bit (INT8 codes included)
    over = {"N": 8192 + 100, "Hq": 4, "Hkv": 1} if name == "llm_128k" else {}
    w, t = workload(name, **over)
    p = params_for(w)
    q, k = to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, q, k)
    ws2 = fb.workspace(p, dev())
    m2, i2, c2, sq2, sk2 = fb.predict_outputs(p, dev())
    fb.sparge_predict_pool(p, q, k, ws2)
    fb.sparge_predict_select(p, m2, i2, c2, sq2, sk2, ws2)
    torch.cuda.synchronize()
    assert torch.equal(mask, m2) and torch.equal(cnt, c2)
    assert torch.equal(sq, sq2) and torch.equal(sk, sk2)
    for r in range(cnt.numel()):
        n = int(cnt.view(-1)[r])
        assert torch.equal(idx.view(-1, idx.shape[-1])[r, :n], i2.view(-1, i2.shape[-1])[r, :n])
    if w.qk_int8:
        reg = ws_regions(p)
        a, b = reg["q_codes"], reg["kbar"] + 4 * p.B * p.Hkv * p.d
        assert torch.equal(ws[a:b], ws2[a:b])
        Tn = -(-p.N // p.bk)
        a, b = reg["k_sum64"], reg["k_sum64"] + 8 * p.B * p.Hkv * Tn * p.d
        assert torch.equal(ws[a:b], ws2[a:b])


@pytest.mark.parametrize("tau,theta", [(1.0, 0.5), (0.3, -1.5), (0.5, 1.5), (0.7, 0.0)])
def test_predict_hyperparameter_limits(tau, theta):
    # tau = 1 keeps every finite block, theta > 1 makes every block a fix
    # block, theta < -1 is pure TopCdf
    w, t = workload("llm_32k", N=4096, Hq=4, Hkv=2)
    Q, K, _ = oracle_inputs(w, t)
    p = params_for(w, tau=tau, theta=theta)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype))
    pr = orc.predict_mask(Q, K, w.bq, w.bk, tau, theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    check_mask(M, pr, f"llm 4K tau {tau} theta {theta}")
    if theta > 1:
        assert np.array_equal(M[0, 0], pr["visible"])


# ----------------------------------------------------------------------------
# stage 2: attention on the oracle's mask
# ----------------------------------------------------------------------------

def _attention_case(name, over, tiles_per_head=None, heads=None, **pkw):
    w, t = workload(name, **over)
    Q, K, V = oracle_inputs(w, t)
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    io, co = orc.mask_compact(pr["M"])
    p = params_for(w, **pkw)
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    ws = None
    if w.qk_int8:
        # the INT8 codes are written by the predictor into the workspace the
        # attention then reads
        ws = gpu_predict(p, q, k)[0]
    idx, cnt = gpu_compact(p, pr["M"])
    o, st = gpu_attention(p, q, k, v, idx, cnt, ws)
    tiles = None
    if tiles_per_head is not None:
        tiles = sample_tiles(w, tiles_per_head, heads, needles=t["needles"])
    O, ost = orc.sparse_attention(Q, K, V, io, co, w.bq, w.bk, pkw.get("lam", w.lam), w.causal,
                                  w.scale, tiles=tiles)
    rows = tile_rows(w, tiles) if tiles is not None else None
    return w, o.cpu().numpy(), O, ost, st, rows


ATTN_CASES = [("tiny", {}, None, None), ("image_dit", {}, None, None),
              ("video_dit", {}, 2, [0, 11, 23]), ("llm_32k", {}, 2, [0, 5, 17, 31])]


@pytest.mark.parametrize("name,over,tph,heads", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_attention_fp32_output_matches_oracle(name, over, tph, heads):
    w, o, O, ost, st, rows = _attention_case(name, over, tph, heads)
    # a lambda decision within 1e-3 of the threshold may flip in float32 and
    # move a whole 32-row slice: those rows are reported, not compared
    report_lambda(ost, name, rows)
    mx, l1 = compare_rows(o, O, rows, exclude=ost["near_rows"])
    assert mx <= MAX_ABS and l1 <= MEAN_REL_L1, (mx, l1, ost["near_lambda"])
    if rows is None:
        # every tile evaluated: the work counters match the oracle's exactly
        assert st[1] == ost["qk_blocks"]
        assert abs(int(st[4]) - ost["skipped_slices"]) <= ost["near_lambda"]


@pytest.mark.parametrize("name", ["llm_32k", "llm_128k"])
def test_batched_gqa_with_ragged_tail(name):
    # B = 2, GQA 2:1 and a ragged last block: the tile, batch and KV-head
    # indexing of every kernel (pooling, select, attention's KV-head-major tile
    # order) across batches, in 16-bit and INT8 modes, against the oracle
    over = dict(N=2048 + 40, B=2, Hq=4, Hkv=2)
    w, t = workload(name, **over)
    Q, K, _ = oracle_inputs(w, t)
    p = params_for(w)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype))
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    check_mask(M, pr, f"{name} B2 ragged")
    assert np.abs(sq.cpu().numpy() - pr["s_q"]).max() < 1e-5
    check_pooled_means(ws, p, pr)
    w, o, O, ost, st, rows = _attention_case(name, over)
    if w.qk_int8:
        l1 = np.abs(o - O).sum() / np.abs(O).sum()
        cos = (o * O).sum() / np.linalg.norm(o) / np.linalg.norm(O)
        assert l1 <= INT8_REL_L1 and cos >= INT8_COS, (l1, cos)
    else:
        mx, l1 = compare_rows(o, O, rows, exclude=ost["near_rows"])
        assert mx <= MAX_ABS and l1 <= MEAN_REL_L1, (mx, l1, ost["near_lambda"])
        assert st[1] == ost["qk_blocks"]
    # the two batches differ, and so must their outputs
    assert not np.allclose(o[0], o[1])


def test_attention_16bit_output_is_rounded_fp32_result():
    # the 16-bit output mode differs from the float32 mode only in the
    # epilogue store: it must be exactly the round-to-nearest-even of the
    # float32 result, and within the absolute bar plus half an ulp of the
    # oracle
    from gpu_common import TD
    for name in ("tiny", "image_dit"):
        w, t = workload(name)
        Q, K, V = oracle_inputs(w, t)
        pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
        io, co = orc.mask_compact(pr["M"])
        q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
        p16 = params_for(w, o_dtype=TD[w.dtype])
        p32 = params_for(w)
        idx, cnt = gpu_compact(p16, pr["M"])
        o16, _ = gpu_attention(p16, q, k, v, idx, cnt, out_dtype=TD[w.dtype])
        o32, _ = gpu_attention(p32, q, k, v, idx, cnt)
        assert torch.equal(o16, o32.to(TD[w.dtype]))
        O, ost = orc.sparse_attention(Q, K, V, io, co, w.bq, w.bk, w.lam, w.causal, w.scale)
        g = o16.float().cpu().numpy().astype(np.float64)
        half_ulp = np.abs(O) * (2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -11)
        keep = ~ost["near_rows"][..., None]
        assert np.all((np.abs(g - O) <= MAX_ABS + half_ulp) | ~keep)


@pytest.mark.parametrize("name,over", [("tiny", {}), ("image_dit", {"Hq": 4, "Hkv": 4}),
                                       ("video_dit", {"Hq": 2, "Hkv": 2}),
                                       ("llm_32k", {"N": 4096, "Hq": 8, "Hkv": 2}),
                                       ("llm_32k", {"N": 1000, "Hq": 4, "Hkv": 1, "B": 2})])
def test_dense_limit_equals_torch_softmax_attention(name, over):
    # theta > 1 makes every block a fix block and lambda = -inf skips nothing:
    # the result is plain softmax attention
    w, t = workload(name, **over)
    p = params_for(w, theta=2.0, lam=float("-inf"))
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    ws, mask, idx, cnt, _, _ = gpu_predict(p, q, k)
    o, st = gpu_attention(p, q, k, v, idx, cnt, ws)
    ref = torch_dense_attention(q, k, v, w.scale, w.causal)
    err = (o - ref).abs()
    assert err.max().item() <= MAX_ABS
    assert (err.sum() / ref.abs().sum()).item() <= MEAN_REL_L1
    assert st[4] == 0


# ----------------------------------------------------------------------------
# INT8 Q K^T with K smoothing
# ----------------------------------------------------------------------------

def int8_state(ws, p, shape_q, shape_k):
    """The predictor's INT8 outputs read back from the workspace: Q and K
    codes, their block scales and kbar."""
    reg = ws_regions(p)
    raw = ws.cpu().numpy()
    Tm, Tn = -(-p.N // p.bq), -(-p.N // p.bk)
    take = lambda name, n, dt: raw[reg[name]:reg[name] + n * np.dtype(dt).itemsize].view(dt)
    return {"q_codes": take("q_codes", int(np.prod(shape_q)), np.int8).reshape(shape_q),
            "k_codes": take("k_codes", int(np.prod(shape_k)), np.int8).reshape(shape_k),
            "dq": take("dq", p.B * p.Hq * Tm, np.float32).reshape(p.B, p.Hq, Tm),
            "dk": take("dk", p.B * p.Hkv * Tn, np.float32).reshape(p.B, p.Hkv, Tn),
            "kbar": take("kbar", p.B * p.Hkv * p.d, np.float32).reshape(p.B, p.Hkv, p.d)}


def check_int8_state(ws, p, Q, K):
    """Algorithm 1 step 2: every code, block scale and the K mean are integer
    or float32 decisions both sides take the same way, so they must match the
    oracle bit for bit."""
    g = int8_state(ws, p, Q.shape, K.shape)
    qt = orc.quantize_qk(Q.astype(np.float32), K.astype(np.float32), p.bq, p.bk)
    assert np.array_equal(g["kbar"], qt["kbar"]), np.abs(g["kbar"] - qt["kbar"]).max()
    assert np.array_equal(g["dq"], qt["dq"]) and np.array_equal(g["dk"], qt["dk"])
    nq = int((g["q_codes"] != qt["q_codes"]).sum())
    nk = int((g["k_codes"] != qt["k_codes"]).sum())
    print(f"[int8 N={p.N}] codes differing: Q {nq} of {Q.size}, K {nk} of {K.size}")
    assert nq == 0 and nk == 0


def check_pooled_means(ws, p, pr):
    """Eq. 4-5: the float32 block means the predictor keeps in its workspace
    against the oracle's float64 means (relative to the block's scale)."""
    reg = ws_regions(p)
    raw = ws.cpu().numpy()
    Tm, Tn = -(-p.N // p.bq), -(-p.N // p.bk)
    qm = raw[reg["q_mean"]:reg["q_mean"] + 4 * p.B * p.Hq * Tm * p.d].view(np.float32)
    km = raw[reg["k_mean"]:reg["k_mean"] + 4 * p.B * p.Hkv * Tn * p.d].view(np.float32)
    for name, got, ref in (("q", qm, pr["q"]), ("k", km, pr["k"])):
        ref = ref.reshape(-1, p.d)
        got = got.reshape(-1, p.d).astype(np.float64)
        scale = np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-3)
        err = float((np.abs(got - ref) / scale).max())
        assert err < 2e-6, (name, err)


def test_int8_codes_and_scales_match_oracle():
    w, t = workload("llm_128k", N=4096, Hq=8, Hkv=2)
    Q, K, _ = oracle_inputs(w, t)
    p = params_for(w)
    ws, *_ = gpu_predict(p, to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype))
    check_int8_state(ws, p, Q, K)
    check_pooled_means(ws, p, orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal,
                                               w.scale))


def test_int8_codes_exact_at_full_length():
    """The 128K workload: every Q and K code, every scale and kbar."""
    w, t = workload("llm_128k")
    Q, K, _ = oracle_inputs(w, t)
    p = params_for(w)
    ws, *_ = gpu_predict(p, to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype))
    check_int8_state(ws, p, Q, K)


def test_int8_codes_on_half_integer_quotients():
    """Blocks built so that x / delta is exactly a half-integer for every
    element: head 0 has absmax 127 (delta = 1) and values k + 1/2, head 1 the
    same divided by 8 (delta = 1/8).  Every code takes the division's
    round-half-even (the kernels' exact path); K - kbar is arbitrary float32."""
    rng = np.random.default_rng(3)
    B, H, N, d = 1, 2, 512, 128
    x = rng.integers(-126, 126, size=(B, H, N, d)).astype(np.float32) + np.float32(0.5)
    x[..., ::128, 0] = 127.0                      # absmax of every Q block
    x[:, 1] /= 8
    q16 = x.astype(np.float16)                    # all exact in fp16
    assert np.array_equal(q16.astype(np.float32), x)
    w, _ = workload("llm_128k", N=N, Hq=2, Hkv=2, dtype="f16")
    p = params_for(w)
    qd = torch.from_numpy(q16).to(dev())
    ws, *_ = gpu_predict(p, qd, qd)
    Q = q16.astype(np.float64)
    check_int8_state(ws, p, Q, Q)


def test_int8_state_with_bf16_subnormal_keys():
    """K values that are bf16 subnormals (below 2^-126), zero blocks and
    normal values side by side: kbar is the float64 mean of every token,
    rounded once, with no value flushed to zero; every code and scale
    matches the oracle bit for bit (a subnormal delta takes the exact
    division)."""
    g = torch.Generator().manual_seed(11)
    B, H, N, d = 1, 2, 1024 + 64, 128
    q = torch.randn(B, H, N, d, generator=g)
    k = torch.randn(B, H, N, d, generator=g)
    k[:, 0] *= 2.0 ** -124                        # about a quarter below 2^-126
    k[:, 1, ::7] *= 2.0 ** -130                   # subnormal tokens among normal ones
    k[:, 1, 64:128] = 0.0                         # a whole key block of zeros
    q[:, 1, 128:256] = 0.0                        # a whole query block of zeros
    q16, k16 = q.to(torch.bfloat16), k.to(torch.bfloat16)
    ksub = k16[:, 0].float().abs()
    assert ((ksub > 0) & (ksub < 2.0 ** -126)).float().mean() > 0.1
    w, _ = workload("llm_128k", N=N, Hq=H, Hkv=H)
    p = params_for(w)
    ws, *_ = gpu_predict(p, q16.to(dev()), k16.to(dev()))
    Q, K = q16.double().numpy(), k16.double().numpy()
    check_int8_state(ws, p, Q, K)


def test_int8_with_fp16_io_and_ragged_tail():
    # INT8 Q K^T with fp16 inputs (no V conversion) and a ragged tail: Q codes
    # and scales bit-exact, the mask against the oracle, the output within the
    # INT8 bar
    over = {"N": 2048 + 96, "Hq": 4, "Hkv": 2, "dtype": "f16"}
    w, t = workload("llm_128k", **over)
    Q, K, _ = oracle_inputs(w, t)
    p = params_for(w)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype))
    check_int8_state(ws, p, Q, K)
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    check_mask(mask.cpu().numpy().astype(bool), pr, "int8 f16 ragged")
    w, o, O, ost, st, rows = _attention_case("llm_128k", over)
    l1 = np.abs(o - O).sum() / np.abs(O).sum()
    cos = (o * O).sum() / np.linalg.norm(o) / np.linalg.norm(O)
    assert l1 <= INT8_REL_L1 and cos >= INT8_COS, (l1, cos)


def test_int8_attention_small_matches_exact_scores():
    w, t = workload("llm_128k", N=4096, Hq=8, Hkv=2)
    w_, o, O, ost, st, rows = _attention_case("llm_128k", {"N": 4096, "Hq": 8, "Hkv": 2})
    l1 = np.abs(o - O).sum() / np.abs(O).sum()
    cos = (o * O).sum() / np.linalg.norm(o) / np.linalg.norm(O)
    assert l1 <= INT8_REL_L1 and cos >= INT8_COS, (l1, cos)


def test_int8_attention_full_128k_sampled_tiles():
    w, o, O, ost, st, rows = _attention_case("llm_128k", {}, 1, [0, 13, 31])
    sel = rows
    a, b = o[sel].astype(np.float64), O[sel]
    l1 = np.abs(a - b).sum() / np.abs(b).sum()
    cos = (a * b).sum() / np.linalg.norm(a) / np.linalg.norm(b)
    assert l1 <= INT8_REL_L1 and cos >= INT8_COS, (l1, cos)


# ----------------------------------------------------------------------------
# sparse masks at scale: the block skipping the method exists for
# ----------------------------------------------------------------------------

SPARSE_CASES = [
    # workload, shape overrides, hyper-parameters, sampled tiles per head, heads
    ("llm_32k", {}, {"theta": -1.0, "tau": 0.5}, 2, [0, 9, 31]),
    ("video_dit", {}, {"theta": 0.3}, 2, [0, 12, 23]),
    ("llm_128k", {}, {"theta": -1.0, "tau": 0.5}, 1, [0, 31]),
]


@pytest.mark.parametrize("name,over,hp,tph,heads", SPARSE_CASES,
                         ids=["llm_32k-tau0.5", "video_dit-theta0.3", "llm_128k-int8-tau0.5"])
def test_sparse_mask_attention_at_scale(name, over, hp, tph, heads):
    """Eq. 2 of the paper review: Q_i K_j^T and P~_ij V_j are skipped where
    M_g = 0.  With theta low enough that blocks are selective, TopCdf drops a
    large share of them.  Checked: the GPU mask against the oracle's; the
    attention on the oracle's mask at sampled tiles against the oracle; and
    the whole GPU path (its own mask and skip list) against the oracle's
    attention on that mask.  INT8 runs are held to the INT8 bars against the
    exact-score oracle."""
    w0, t = workload(name, **over)
    w = w0.replace(**hp)
    Q, K, V = oracle_inputs(w, t)
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    if w.grid:
        perm = orc.hilbert_permutation(w.N, w.prefix_len, *w.grid)
        Q, K, V = (orc.permute_tokens(x, perm) for x in (Q, K, V))
        pt = torch.from_numpy(perm.astype(np.int32)).to(dev())
        q, k, v = _permuted(q, pt), _permuted(k, pt), _permuted(v, pt)
    p = params_for(w)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, q, k)
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    cm = check_mask(M, pr, f"{name} {hp}")
    sparsity = 1.0 - M.sum() / cm["visible"]
    print(f"[sparse {name} {hp}] M_g sparsity {sparsity:.3f}")
    assert sparsity > 0.15
    tiles = sample_tiles(w, tph, heads, needles=t["needles"])
    rows = tile_rows(w, tiles)
    for label, Mx, ix, cx in (("oracle mask", pr["M"], *gpu_compact(p, pr["M"])),
                              ("GPU mask", M, idx, cnt)):
        o, st = gpu_attention(p, q, k, v, ix, cx, ws)
        io, co = orc.mask_compact(Mx)
        O, ost = orc.sparse_attention(Q, K, V, io, co, w.bq, w.bk, w.lam, w.causal, w.scale,
                                      tiles=tiles)
        on = o.cpu().numpy()
        assert st[1] == int(Mx.sum())           # one Q K^T product per kept block
        if w.qk_int8:
            a, b = on[rows].astype(np.float64), O[rows]
            l1 = np.abs(a - b).sum() / np.abs(b).sum()
            cos = (a * b).sum() / np.linalg.norm(a) / np.linalg.norm(b)
            print(f"[sparse {name} {label}] INT8 rel L1 {l1:.2e} cos {cos:.6f}")
            assert l1 <= INT8_REL_L1 and cos >= INT8_COS, (label, l1, cos)
        else:
            report_lambda(ost, f"{name} {label}", rows)
            mx, l1 = compare_rows(on, O, rows, exclude=ost["near_rows"])
            print(f"[sparse {name} {label}] max|dO| {mx:.2e} rel L1 {l1:.2e}")
            assert mx <= MAX_ABS and l1 <= MEAN_REL_L1, (label, mx, l1)


def _permuted(x, pt):
    y = torch.empty_like(x)
    fb.sparge_hilbert_permute(x, y, pt)
    return y


# ----------------------------------------------------------------------------
# edge cases
# ----------------------------------------------------------------------------

def test_maximum_length_mask_and_sampled_tiles():
    # the largest N the library accepts (5952 key blocks of 64, the select
    # kernel's shared-memory bound), causal, one head: the whole mask against
    # the oracle, attention on sampled tiles including the last (5952 blocks)
    N = 5952 * 64
    w, t = workload("llm_32k", N=N, Hq=1, Hkv=1)
    Q, K, _ = oracle_inputs(w, t)
    p = params_for(w)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, to_dev(t["q"], w.dtype), to_dev(t["k"], w.dtype))
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    check_mask(M, pr, "maximum length")
    assert int(cnt.view(-1)[-1]) == M[0, 0, -1].sum() == 5952
    w, o, O, ost, st, rows = _attention_case("llm_32k", {"N": N, "Hq": 1, "Hkv": 1}, 2, [0])
    report_lambda(ost, "maximum length", rows)
    mx, l1 = compare_rows(o, O, rows, exclude=ost["near_rows"])
    assert mx <= MAX_ABS and l1 <= MEAN_REL_L1, (mx, l1, ost["near_lambda"])
    # one more key block is refused before anything runs
    assert fb.sparge_workspace_bytes(params_for(w.replace(N=N + 1))) == 0


def test_maximum_length_selective_rows_and_constant_scores():
    """The TopCdf radix select on the longest rows the library accepts (5952
    key blocks): theta = -1 makes every query block selective and tau = 0.5
    makes TopCdf cut.  Head 1 has Q = 0, so every score of its rows is equal
    and every weight is 1: the histogram's largest bucket sums (5952 weights
    of 2^38 in two 32-bit halves) and TopCdf's ties (all entries equal the cut
    value, so all are kept, Eq. 8's reading)."""
    N = 5952 * 64
    w, t = workload("llm_32k", N=N, Hq=2, Hkv=1)
    w = w.replace(theta=-1.0, tau=0.5)
    q = t["q"].copy()
    q[:, 1] = 0
    Q, K = to_f64(q, w.dtype), to_f64(t["k"], w.dtype)
    p = params_for(w)
    ws, mask, idx, cnt, sq, sk = gpu_predict(p, to_dev(q, w.dtype), to_dev(t["k"], w.dtype))
    pr = orc.predict_mask(Q, K, w.bq, w.bk, w.tau, w.theta, w.causal, w.scale)
    M = mask.cpu().numpy().astype(bool)
    check_mask(M, pr, "maximum length, theta -1, tau 0.5")
    vis = pr["visible"]
    assert np.array_equal(M[0, 1], vis)          # constant rows keep every visible block
    assert M[0, 0].sum() < 0.9 * vis.sum()       # selective rows drop blocks
    assert int(cnt.view(-1)[-1]) == M[0, 1, -1].sum() == 5952


@pytest.mark.parametrize("N,causal", [(1, False), (1, True), (65, True), (129, False),
                                      (200, True), (1000, False)])
def test_ragged_and_tiny_lengths(N, causal):
    w, t = workload("llm_32k", N=max(N, 256), Hq=2, Hkv=1)
    sl = lambda a: np.ascontiguousarray(a[:, :, :N])
    q, k, v = (to_dev(sl(t[x]), w.dtype) for x in ("q", "k", "v"))
    w = w.replace(N=N, causal=causal)
    p = params_for(w, theta=2.0, lam=float("-inf"))
    ws, mask, idx, cnt, _, _ = gpu_predict(p, q, k)
    o, _ = gpu_attention(p, q, k, v, idx, cnt, ws)
    ref = torch_dense_attention(q, k, v, w.scale, causal)
    assert (o - ref).abs().max().item() <= MAX_ABS


def test_empty_rows_and_custom_masks():
    # tiles with an empty skip list output 0; fully-future blocks kept by a
    # custom mask contribute nothing; rows that see no key output 0
    w, t = workload("llm_32k", N=512, Hq=2, Hkv=1)
    Q, K, V = oracle_inputs(w, t)
    M = np.zeros((1, 2, 4, 8), dtype=bool)
    M[0, 0, 1, :] = True          # includes future blocks 4..7 for tile 1
    M[0, 0, 2, 3] = True
    M[0, 1, 3, [1, 6]] = True
    M[0, 1, 0, 1] = True          # rows 0..63 see no key of block 1
    p = params_for(w, lam=float("-inf"))
    idx, cnt = gpu_compact(p, M)
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    o, _ = gpu_attention(p, q, k, v, idx, cnt)
    io, co = orc.mask_compact(M)
    O, ost = orc.sparse_attention(Q, K, V, io, co, 128, 64, -np.inf, True, w.scale)
    on = o.cpu().numpy()
    assert np.all(on[0, 0, :128] == 0) and np.all(on[0, 1, :64] == 0)
    assert np.abs(on - O).max() <= MAX_ABS


def test_lambda_near_zero_skips_all_but_leading_blocks():
    """lambda = -0.05 skips P~V for every slice whose block maximum is not
    within 0.05 of its running maximum (Eq. 3): most slices of most blocks.
    Outside the rows of decisions within 1e-3 of the threshold (excluded and
    counted) the output meets the same bars as everywhere else."""
    lam = -0.05
    _, o, O, ost, st, _ = _attention_case("llm_32k", {"N": 2048, "Hq": 2, "Hkv": 1}, lam=lam)
    assert st[4] > st[3] and abs(int(st[4]) - ost["skipped_slices"]) <= ost["near_lambda"]
    report_lambda(ost, "lambda -0.05")
    mx, l1 = compare_rows(o, O, exclude=ost["near_rows"])
    assert mx <= MAX_ABS and l1 <= MEAN_REL_L1, (mx, l1, ost["near_lambda"])


def test_empty_problems_are_no_ops():
    w, t = workload("tiny")
    for kw in (dict(N=0), dict(B=0)):
        ww = w.replace(**kw)
        p = params_for(ww)
        ws = torch.zeros(max(256, fb.sparge_workspace_bytes(p)), dtype=torch.uint8, device=dev())
        dummy = torch.zeros(16, dtype=torch.float16, device=dev())
        di = torch.zeros(16, dtype=torch.int32, device=dev())
        fb.sparge_attn_fwd(p, dummy, dummy, dummy, di, di, dummy, ws)
        fb.sparge_predict_mask(p, dummy, dummy, di, di, di, None, None, ws)
    torch.cuda.synchronize()


def test_binding_refuses_buffers_the_parameters_do_not_fit():
    """The C entry points take bare pointers; the binding checks every tensor
    against the sizes, element types and device the parameters imply, so an
    undersized or mistyped buffer raises instead of being read or written out
    of bounds."""
    w, t = workload("tiny")
    p = params_for(w)
    q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
    ws = fb.workspace(p, dev())
    mask, idx, cnt, s_q, s_k = fb.predict_outputs(p, dev())
    o = torch.empty(q.shape, dtype=torch.float32, device=dev())     # o_dtype is f32 here
    bad = [
        # an fp16 O buffer for an f32 output would take half the bytes written
        lambda: fb.sparge_attn_fwd(p, q, k, v, idx, cnt, torch.empty_like(q), ws),
        lambda: fb.sparge_predict_mask(p, q[:, :, :10].contiguous(), k, mask, idx, cnt, None,
                                       None, ws),
        lambda: fb.sparge_predict_mask(p, q, k, mask[..., :1].contiguous(), idx, cnt, None, None,
                                       ws),
        lambda: fb.sparge_predict_mask(p, q, k, mask, idx.float(), cnt, None, None, ws),
        lambda: fb.sparge_predict_mask(p, q.float(), k, mask, idx, cnt, None, None, ws),
        lambda: fb.sparge_predict_select(p, mask, idx, cnt[..., :1].contiguous(), None, None, ws),
        lambda: fb.sparge_attn_fwd(p, q, k, v[:, :, :5].contiguous(), idx, cnt, o, ws),
        lambda: fb.sparge_attn_fwd(p, q, k, v, idx, cnt, o[:, :, :5].contiguous(), ws),
        lambda: fb.sparge_attn_fwd(p, q, k, v, idx, cnt, o, ws,
                                   torch.zeros(2, dtype=torch.int64, device=dev())),
        lambda: fb.sparge_hilbert_permute(q, torch.empty_like(q),
                                          torch.zeros(3, dtype=torch.int32, device=dev())),
        lambda: fb.sparge_hilbert_permute(q, torch.empty_like(q),
                                          torch.zeros(w.N, dtype=torch.int64, device=dev())),
        lambda: fb.sparge_attn_fwd(p, q, k, v, idx, cnt, o.cpu(), ws),
    ]
    for call in bad:
        with pytest.raises(fb.SpargeError) as e:
            call()
        assert e.value.code == 1
    torch.cuda.synchronize()
    # the well-formed call still runs
    fb.sparge_predict_mask(p, q, k, mask, idx, cnt, s_q, s_k, ws)
    fb.sparge_attn_fwd(p, q, k, v, idx, cnt, o, ws)
    torch.cuda.synchronize()
