"""CPU oracle for the hybrid compressed-attention hot path (CSA / HCA).

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, FP64 statement of
what the library computes.  Only the tests, the smoke check and the bench's
CPU-baseline leg may import it; the product path never does.  It shares no
code with the CUDA library.

Sources (web pages about DeepSeek-V4):
  [p1] "DeepSeek V4的4个技巧", section 1 "技巧1：混合注意力"
  [p2] "深度解析 DeepSeek-V4：百万级长文本的低成本突破", sections
       "CSA：Compressed Sparse Attention" (Step 1 Compress, Step 2 Select, the
       ASCII figure), "HCA：Heavily Compressed Attention",
       "Sliding Window Branch", "Attention Sink"
  [p3] untitled classical-Chinese paraphrase page, the sentences headed
       "Partial RoPE", "Attention sink", "第一步，KV压缩", "第二步，lightning
       indexer + top-k选择", "第三步，core attention" and the strict-causality,
       HCA-no-overlap and sliding-window sentences
  [p4] "DeepSeek V4 技术架构深度解析", section "二、CSA + HCA"

Readings of points the pages leave open:
  * gate granularity: one softmax over the window's tokens per channel; a
    per-token gate is the broadcast case;
  * the CSA window of entry j is the 2m tokens [(j-1)m, (j+1)m) clipped at 0,
    the HCA window is [j m', (j+1) m'); an entry exists only for complete
    own-blocks, so there are floor(T/m) of them;
  * entry j is visible to the query at position t iff j < floor(t/m);
  * indexer score s[t,j] = sum_h w[t,h] * relu(q_I[t,h] . k_I[j]), no scale;
  * top-k: the k largest scores among the visible entries, ties to the lower
    index, indices emitted ascending, -1 padded;
  * RoPE on the last R dims, adjacent pairs (2i, 2i+1) of that slice,
    theta_i = base^(-2i/R); compressed entry j sits at position j*m, raw token
    s at position s; the rotated entry is both key and value; the output's
    rotary slice is rotated back by -t;
  * logits scale 1/sqrt(D); window = raw tokens s with t-W < s <= t;
    sink = one logit per head added as exp(sigma_h) to the denominator.
  * FP4 indexer path: MXFP4 blocks (32 values, one power-of-two scale with
    exponent floor(log2 amax) - 2, E2M1 codes rounded to nearest even and
    saturated); the query is quantised per (row, head) and the scores use
    the exact dequantised values.
  * grouped output projection: g groups of consecutive heads, each projected
    to d_g, concatenated and projected to d; the intermediate is stored in
    BF16 (the pages give neither g nor d_g);
  * FP8 entry cache: E4M3 for the non-rotary dims with one power-of-two scale
    per entry (largest magnitude mapped to at most 448), rotary dims in BF16.

Parity pins: every function here is checked in tests/test_oracle_pins.py
against closed forms, a library attention routine, brute force and values the
pages print.
"""
import math

import numpy as np

__all__ = [
    "compress", "csa_compress", "hca_compress",
    "n_visible", "indexer_scores", "topk_select", "topk_from_scores", "indexer_topk",
    "rope_rotate", "attend_one", "csa_sparse_attn", "hca_dense_attn",
]


# ----------------------------------------------------------------------------
# Step 1: KV compression  ([p2] CSA Step 1: m consecutive tokens are merged into
# one entry with learned softmax weights; [p3] "第一步，KV压缩" and the sentence on
# an attention-like pooling with learned weights; [p3] the sentence saying HCA
# pools every m' tokens without CSA's overlap)
# ----------------------------------------------------------------------------
def compress(kv, gate, m, window, rms_weight=None, rms_eps=1e-6):
    """Pool a [T, D] token sequence into floor(T/m) entries.

    Entry j pools the tokens [(j+1)m - window, (j+1)m) clipped at 0 with
    softmax weights taken over those tokens, separately for every channel:
        c[j,d] = sum_i softmax_i(gate[i,d]) * kv[i,d].
    gate may be [T, D] (per channel) or [T] (one logit per token).
    With rms_weight, c[j] is RMS-normalised and scaled ([p2] "Attention Sink"
    section, last paragraph: RMSNorm on the compressed KV entries).
    """
    kv = np.asarray(kv, dtype=np.float64)
    gate = np.asarray(gate, dtype=np.float64)
    T, D = kv.shape
    if gate.ndim == 1:
        gate = np.repeat(gate[:, None], D, axis=1)
    Nc = T // m
    out = np.zeros((Nc, D), dtype=np.float64)
    for j in range(Nc):
        hi = (j + 1) * m
        lo = max(0, hi - window)
        g = gate[lo:hi]
        e = np.exp(g - g.max(axis=0, keepdims=True))
        wts = e / e.sum(axis=0, keepdims=True)
        out[j] = (wts * kv[lo:hi]).sum(axis=0)
    if rms_weight is not None:
        rms = np.sqrt(np.mean(out * out, axis=1, keepdims=True) + rms_eps)
        out = out / rms * np.asarray(rms_weight, dtype=np.float64)[None, :]
    return out


def csa_compress(kv, gate, m=4, rms_weight=None, rms_eps=1e-6):
    """CSA: overlapping 2m window with stride m."""
    return compress(kv, gate, m, 2 * m, rms_weight, rms_eps)


def hca_compress(kv, gate, m=128, rms_weight=None, rms_eps=1e-6):
    """HCA: non-overlapping blocks of m tokens."""
    return compress(kv, gate, m, m, rms_weight, rms_eps)


def n_visible(t, m, n_c):
    """Compressed entries visible to the query at absolute position t:
    j < floor(t/m) ([p3] strict causality: a query does not see the other
    tokens of its own compressed block)."""
    return int(max(0, min(n_c, t // m)))


# ----------------------------------------------------------------------------
# Step 2: Lightning Indexer + top-k  ([p2] CSA Step 2 "Select" and the ASCII
# figure; [p3] "第二步，lightning indexer + top-k选择" and the sentence on a
# light indexer scoring every compressed block against each query token)
# ----------------------------------------------------------------------------
def indexer_scores(q_idx, w, k_idx, q_pos0, m):
    """Scores [Tq, Nc] in FP64; entries that are not visible are -inf.

    s[t,j] = sum_h w[t,h] * max(0, q_I[t,h,:] . k_I[j,:]).
    """
    q_idx = np.asarray(q_idx, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k_idx = np.asarray(k_idx, dtype=np.float64)
    Tq = q_idx.shape[0]
    Nc = k_idx.shape[0]
    s = np.full((Tq, Nc), -np.inf, dtype=np.float64)
    for i in range(Tq):
        nv = n_visible(q_pos0 + i, m, Nc)
        if nv == 0:
            continue
        dots = q_idx[i] @ k_idx[:nv].T           # [H_I, nv]
        s[i, :nv] = w[i] @ np.maximum(dots, 0.0)
    return s


def topk_select(row, k):
    """Indices of the k largest values of `row` (ties to the lower index),
    returned ascending and padded with -1 to length k."""
    row = np.asarray(row, dtype=np.float64)
    assert not np.isnan(row).any(), "NaN score"
    n = row.shape[0]
    j = np.arange(n)
    order = np.lexsort((j, -row))               # primary: score descending; then index ascending
    chosen = np.sort(order[:min(k, n)])
    out = np.full(k, -1, dtype=np.int64)
    out[:chosen.shape[0]] = chosen
    return out


def topk_from_scores(scores, n_valid, k):
    """Row-wise selection over the first n_valid[r] columns of each row."""
    scores = np.asarray(scores)
    out = np.full((scores.shape[0], k), -1, dtype=np.int64)
    for r in range(scores.shape[0]):
        nv = int(n_valid[r])
        if nv > 0:
            out[r] = topk_select(scores[r, :nv], k)
    return out


def indexer_topk(q_idx, w, k_idx, q_pos0, m, k, score_dtype=np.float32):
    """Scores in FP64, rounded to the selection precision (FP32, the kernel's),
    then the top-k of the visible prefix of every row."""
    s = indexer_scores(q_idx, w, k_idx, q_pos0, m)
    Tq, Nc = s.shape
    nv = [n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    s_sel = s.astype(score_dtype).astype(np.float64)
    return topk_from_scores(s_sel, nv, k), s


# ----------------------------------------------------------------------------
# FP4 indexer QK path  ([p2] "FP4 Quantization-Aware Training": the indexer
# computes its query-key scores in FP4 (E2M1) with block scale factors that a
# wider format absorbs on dequantisation; [p4] "三、FP4量化": the table row that
# takes the CSA indexer QK path from FP32 to FP4; CSA Step 2 "Select": the
# Lightning Indexer runs in FP4 precision)
#
# Block format (the pages name E2M1 with block scales but no block size or
# scale encoding; the plainest reading is the OCP Microscaling MXFP4 format):
# 32 consecutive values share one power-of-two scale 2^X stored as a UE8M0
# byte X + 127; each value is the E2M1 number nearest to x / 2^X.
# ----------------------------------------------------------------------------
MX_BLOCK = 32
# E2M1 magnitudes by 3-bit code (exponent bits e1 e0, mantissa bit m):
# e = 0: m * 0.5 (subnormal); e > 0: (1 + m/2) * 2^(e-1)
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def mx_scale_exponent(amax):
    """Shared exponent of blocks with largest magnitudes `amax` (array):
    X = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent, so amax / 2^X
    lies in [4, 8)), clamped to the UE8M0 range [-127, 127]; an all-zero
    block takes X = -127."""
    amax = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(amax)            # amax = f * 2^e, f in [0.5, 1)
    X = np.clip((e - 1) - 2, -127, 127)
    return np.where(amax == 0.0, -127, X).astype(np.int64)


def e2m1_codes(y):
    """4-bit E2M1 codes of the values nearest to y (array): round to nearest,
    ties to the code with an even mantissa bit (code bit 0), magnitudes above
    6 saturate to 6; bit 3 is the sign of y."""
    y = np.asarray(y, dtype=np.float64)
    d = np.abs(np.abs(y)[..., None] - E2M1_VALUES)          # distance to each magnitude
    near = d == d.min(axis=-1, keepdims=True)
    even = near & (np.arange(8) % 2 == 0)
    c = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(near, axis=-1))
    return (c | np.where(y < 0, 8, 0)).astype(np.uint8)


def e2m1_code(y):
    return int(e2m1_codes(np.array([y]))[0])


def quantize_mxfp4(x):
    """MXFP4 of x[..., C] (C a multiple of 32) along the last axis.

    Returns (codes uint8 [..., C/2], scales uint8 [..., C/32]): byte i of a
    row's codes holds element 2i in its low nibble and 2i+1 in its high
    nibble; a block holding a non-finite value gets scale byte 255 and zero
    codes."""
    x = np.asarray(x, dtype=np.float64)
    C = x.shape[-1]
    assert C % MX_BLOCK == 0
    rows = x.size // C if C else 0
    if rows > 8192:                   # bound the temporaries: quantise in row slices
        flat = x.reshape(rows, C)
        parts = [quantize_mxfp4(flat[r:r + 8192]) for r in range(0, rows, 8192)]
        return (np.concatenate([p[0] for p in parts]).reshape(x.shape[:-1] + (C // 2,)),
                np.concatenate([p[1] for p in parts]).reshape(x.shape[:-1] + (C // MX_BLOCK,)))
    blk = x.reshape(x.shape[:-1] + (C // MX_BLOCK, MX_BLOCK))
    finite = np.isfinite(blk).all(axis=-1)
    amax = np.where(finite, np.abs(np.where(np.isfinite(blk), blk, 0.0)).max(axis=-1), 0.0)
    X = mx_scale_exponent(amax)
    y = np.ldexp(np.where(np.isfinite(blk), blk, 0.0), -X[..., None])   # exact: a power-of-two scaling
    c = np.where(finite[..., None], e2m1_codes(y), 0).astype(np.uint8).reshape(x.shape)
    codes = (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)
    scales = np.where(finite, X + 127, 255).astype(np.uint8)
    return codes, scales


def dequantize_mxfp4(codes, scales):
    """Exact values (FP64) of MXFP4 codes and scales: E2M1 value times 2^X."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    lo = codes & 0xF
    hi = codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))
    val = E2M1_VALUES[nib & 7] * np.where(nib & 8, -1.0, 1.0)
    X = scales.astype(np.float64) - 127.0
    X = np.where(scales == 255, np.nan, X)
    return val * np.exp2(np.repeat(X, MX_BLOCK, axis=-1))


def indexer_scores_mxfp4(q_idx, w, k_codes, k_scales, q_pos0, m):
    """Indexer scores of the FP4 QK path: the query is quantised to MXFP4 per
    (row, head) and both sides are taken at their exact dequantised values;
    the score formula is the one of indexer_scores."""
    qc, qs = quantize_mxfp4(q_idx)
    return indexer_scores(dequantize_mxfp4(qc, qs), w, dequantize_mxfp4(k_codes, k_scales), q_pos0, m)


def indexer_topk_mxfp4(q_idx, w, k_codes, k_scales, q_pos0, m, k, score_dtype=np.float32):
    """Top-k of the FP4-path scores, rounded to the selection precision."""
    s = indexer_scores_mxfp4(q_idx, w, k_codes, k_scales, q_pos0, m)
    Tq, Nc = s.shape
    nv = [n_visible(q_pos0 + i, m, Nc) for i in range(Tq)]
    return topk_from_scores(s.astype(score_dtype).astype(np.float64), nv, k), s


# ----------------------------------------------------------------------------
# Step 3: core attention  ([p3] "第三步，core attention", "Partial RoPE",
# "Attention sink", the sliding-window sentence; [p2] "Sliding Window Branch",
# "Attention Sink")
# ----------------------------------------------------------------------------
def rope_rotate(x, pos, R, base=10000.0):
    """Rotate the last R dims of x[..., D] by angle pos*theta_i per adjacent
    pair (2i, 2i+1) of that slice, theta_i = base^(-2i/R).  pos broadcasts
    against x's leading dims."""
    x = np.array(x, dtype=np.float64, copy=True)
    if R == 0:
        return x
    D = x.shape[-1]
    i = np.arange(R // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / R)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., D - R::2].copy()
    b = x[..., D - R + 1::2].copy()
    x[..., D - R::2] = a * c - b * s
    x[..., D - R + 1::2] = a * s + b * c
    return x


def attend_one(q_t, t, entries, ckv, m, kv, kv_pos0, W, sink, R, base=10000.0, scale=None):
    """One query position t, all heads.

    Keys (= values): the compressed entries `entries` (each rotated at j*m)
    followed by the raw window tokens s with t-W < s <= t that kv holds
    (rows kv_pos0 .. kv_pos0+len(kv)-1, each rotated at s).  One softmax over
    all of them with exp(sink_h) added to the denominator; the output's rotary
    slice is rotated by -t.  Returns (out [H,D], lse [H]) with
    lse = log(sum exp(logits) + exp(sink)).
    """
    q_t = np.asarray(q_t, dtype=np.float64)
    H, D = q_t.shape
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    entries = np.asarray(entries, dtype=np.int64)
    keys = []
    if entries.size:
        keys.append(rope_rotate(np.asarray(ckv, dtype=np.float64)[entries], entries * m, R, base))
    lo = max(t - W + 1, kv_pos0, 0)
    hi = min(t, kv_pos0 + kv.shape[0] - 1)
    if hi >= lo:
        s = np.arange(lo, hi + 1)
        keys.append(rope_rotate(np.asarray(kv, dtype=np.float64)[s - kv_pos0], s, R, base))
    qr = rope_rotate(q_t, t, R, base)
    sink = None if sink is None else np.asarray(sink, dtype=np.float64)
    if not keys:
        out = np.zeros((H, D))
        lse = np.full(H, -np.inf) if sink is None else sink.copy()
        return out, lse
    K = np.concatenate(keys, axis=0)                 # [n, D]
    logits = scale * (qr @ K.T)                      # [H, n]
    mx = logits.max(axis=1)
    if sink is not None:
        mx = np.maximum(mx, sink)
    e = np.exp(logits - mx[:, None])
    denom = e.sum(axis=1)
    if sink is not None:
        denom = denom + np.exp(sink - mx)
    out = (e @ K) / denom[:, None]
    out = rope_rotate(out, -t, R, base)
    return out, mx + np.log(denom)


def _rows(B, Tq, rows):
    if rows is None:
        return [(b, i) for b in range(B) for i in range(Tq)]
    return list(rows)


def csa_sparse_attn(q, ckv, idx, kv, q_pos0, kv_pos0, m, W, sink, R, base=10000.0,
                    scale=None, rows=None):
    """CSA core attention over the selected entries idx[b,i,:] (>= 0 only).

    q [B,Tq,H,D], ckv [B,Nc,D], idx [B,Tq,k], kv [B,Tkv,D].
    Returns (out [n,H,D], lse [n,H]) for the (b, i) pairs in `rows`
    (all rows when None)."""
    B, Tq = q.shape[0], q.shape[1]
    outs, lses = [], []
    for b, i in _rows(B, Tq, rows):
        sel = np.asarray(idx[b, i])
        sel = sel[sel >= 0]
        assert (sel < ckv.shape[1]).all()
        o, l = attend_one(q[b, i], q_pos0 + i, sel, ckv[b], m, kv[b], kv_pos0, W, sink, R, base, scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def hca_dense_attn(q, ckv, kv, q_pos0, kv_pos0, m, W, sink, R, base=10000.0,
                   scale=None, rows=None):
    """HCA core attention over every visible entry j < floor(t/m)."""
    B, Tq = q.shape[0], q.shape[1]
    Nc = ckv.shape[1]
    outs, lses = [], []
    for b, i in _rows(B, Tq, rows):
        t = q_pos0 + i
        sel = np.arange(n_visible(t, m, Nc))
        o, l = attend_one(q[b, i], t, sel, ckv[b], m, kv[b], kv_pos0, W, sink, R, base, scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


# ----------------------------------------------------------------------------
# Step 4: grouped output projection  ([p3] "第四步，grouped output projection" and
# the sentence explaining it: with head dimension c = 512, projecting all head
# outputs straight back to d would be costly, so the n_h heads are split into g
# groups, each group is first projected to an intermediate width d_g, and the
# concatenated groups are projected back to d; V4-Flash's hidden size is 4096)
# ----------------------------------------------------------------------------
def grouped_out_proj(o, w_group, w_out, round_mid=True):
    """y = W_out . concat_g(W_group[g] . o_g) for every token.

    o       [T, n_h, c]  attention outputs (heads of group g: g*n_h/g .. +n_h/g)
    w_group [g, d_g, (n_h/g)*c]  per-group projection, rows = outputs
    w_out   [d, g*d_g]           merge projection, rows = outputs
    The intermediate group projections are rounded to BF16 when `round_mid`
    (they are stored between the two projections in BF16).  FP64 otherwise.
    """
    o = np.asarray(o, dtype=np.float64)
    w_group = np.asarray(w_group, dtype=np.float64)
    w_out = np.asarray(w_out, dtype=np.float64)
    T, n_h, c = o.shape
    g, d_g, kg = w_group.shape
    assert n_h % g == 0 and kg == (n_h // g) * c and w_out.shape[1] == g * d_g
    x = o.reshape(T, g, kg)
    mid = np.stack([x[:, j, :] @ w_group[j].T for j in range(g)], axis=1).reshape(T, g * d_g)
    if round_mid:
        mid = _round_bf16(mid)
    return mid @ w_out.T


def _round_bf16(x):
    """Nearest BF16 value (8 significant bits, exponent range of FP32; ties to
    even) of each FP64 value: x / ulp(x) rounded half-to-even, times ulp(x)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(np.where(x == 0, 1.0, x))          # |x| = f * 2^e, f in [0.5, 1)
    ulp_exp = np.maximum(e - 8, -133)                    # 8 significant bits; BF16 subnormal spacing 2^-133
    return np.ldexp(np.rint(np.ldexp(x, -ulp_exp)), ulp_exp)


# ----------------------------------------------------------------------------
# FP8 entry cache  ([p4] "KV Cache优化细节": mixed storage, the rotary dims in
# BF16 and the rest in FP8)
#
# Reading (the pages give no FP8 variant or scale): FP8 E4M3 (bias 7, no
# infinities, largest finite 448, subnormals m * 2^-9) for the first D - R dims
# of every entry, with one power-of-two scale per entry 2^X, X the smallest
# integer with max|x| / 2^X <= 448, raised to at least -124 (stored as the
# byte X + 127; an all-zero entry takes X = -124), values rounded to nearest
# even and saturated at 448; the last R (rotary) dims stay BF16.  E4M3 values
# are multiples of 2^-9, so with X >= -124 every E4M3 * 2^X is a multiple of
# 2^-133 (the smallest BF16 subnormal) with at most 4 significant bits: exact
# in BF16, so the cache expands for BF16 tensor cores losslessly.
# ----------------------------------------------------------------------------
def e4m3_value(code):
    """Value of an 8-bit E4M3 code from its fields (sign bit 7, exponent bits
    6-3 with bias 7, mantissa bits 2-0); exponent 0 is subnormal; 0x7F and
    0xFF are NaN."""
    code = int(code)
    sgn = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return sgn * mag


E4M3_POS = np.array([e4m3_value(c) for c in range(0x7F)])     # codes 0x00..0x7E, increasing


def e4m3_codes(y):
    """E4M3 codes of the values nearest to y (array): round to nearest, ties to
    the code with an even mantissa (code bit 0), magnitudes above 448 saturate
    to 448; bit 7 is the sign of y."""
    y = np.asarray(y, dtype=np.float64)
    a = np.minimum(np.abs(y), 448.0)
    hi = np.clip(np.searchsorted(E4M3_POS, a, side="left"), 0, len(E4M3_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - E4M3_POS[lo], E4M3_POS[hi] - a
    c = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    c = np.where(a == E4M3_POS[hi], hi, c)
    return (c | np.where(y < 0, 0x80, 0)).astype(np.uint8)


def quantize_entries_fp8(ckv, R):
    """Entries [..., D] -> (codes uint8 [..., D-R] E4M3, scales uint8 [...]
    (X + 127), rope BF16 values [..., R] as FP64)."""
    x = np.asarray(ckv, dtype=np.float64)
    D = x.shape[-1]
    body, rope = x[..., :D - R], x[..., D - R:]
    amax = np.abs(body).max(axis=-1)
    # smallest X with amax <= 448 * 2^X: with amax = f 2^e (f in [0.5, 1)) and
    # 448 = 0.875 * 2^9, X = e - 9 if f <= 0.875 else e - 8 (exact comparisons)
    f, e = np.frexp(np.where(amax > 0, amax, 1.0))
    X = np.where(f <= 0.875, e - 9, e - 8)
    X = np.where(amax > 0, np.clip(X, -124, 127), -124).astype(np.int64)
    codes = e4m3_codes(np.ldexp(body, -X[..., None]))
    return codes, (X + 127).astype(np.uint8), _round_bf16(rope)


E4M3_ALL = np.array([e4m3_value(c) for c in range(256)])     # value of every code, by e4m3_value


def dequantize_entries_fp8(codes, scales, rope):
    """Exact FP64 entries from the FP8 cache: E4M3 value * 2^X, rotary dims as stored."""
    vals = E4M3_ALL[np.asarray(codes, dtype=np.uint8)]
    X = np.asarray(scales, dtype=np.float64) - 127.0
    return np.concatenate([vals * np.exp2(X)[..., None], np.asarray(rope, dtype=np.float64)], axis=-1)
