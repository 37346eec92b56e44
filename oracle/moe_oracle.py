"""CPU oracle for the forward pass of one FP8 (W8A8 e4m3) mixture-of-experts layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this module: only the
tests, the package smoke check and the benchmark's CPU-baseline leg do. It shares no code with
the CUDA library and imports nothing from it.

What it computes (plain numpy, float64 accumulation, one step after another):

1. router logits  l[t, e] = sum_d x[t, d] * W[e, d] + b[e]
   -- "Routage MoE entre GPU" (viite.ai): the router reads each token's hidden state and scores
      every expert.
2. softmax over all E experts, top-k selection, weights renormalised over the selection
   -- same page: the router keeps the best k (two there) experts and emits one routing weight per
      selection; ELDR (aiweekly.co), third paragraph: outputs equal the standard top-k.
      Exact ties go to the lower expert index.
3. per-token dynamic FP8 activation quantisation (scale = amax / 448)
   -- "La nouvelle bibliotheque megakernel d'Aleph Alpha", W8A8 paragraph: 8-bit weights and
      8-bit activations in the FP8 format.
4. grouping of the routed (token, expert) rows by expert, tokens in ascending order inside a group
   -- "Routage MoE entre GPU": only the selected experts process a token; tokens are dispatched
      to their experts.
5. per routed row: gate/up GEMM on dequantised FP8, SwiGLU, FP8 requantisation of the
   intermediate (per row, over all F), down GEMM
   -- megakernel page, section "Comment fonctionne le megakernel" (expert compute), W8A8.
6. combine: y[t] = sum_j w[t, j] * o[row(t, j)] (+ the shared expert's output, weight 1.0),
   one round-to-nearest-even rounding to bf16, rows back in the original token order
   -- "Routage MoE entre GPU": the two selected outputs are multiplied by their routing weights,
      summed, and the original token order is restored.

Readings where the pages are silent (each listed with its reason in the design notes):
* FP8 = OCP e4m3fn: bias 7, 3 mantissa bits, max 448, no infinities, codes 0x7F/0xFF are NaN;
  encoding rounds to nearest, ties to even, and saturates to +-448.
* Quantisation decisions (the scale amax/448 and the code of value/scale) are taken in fp32 with
  IEEE division, the precision the kernels use; everything else accumulates in float64.
* W13 rows [0, F) are the gate projection, rows [F, 2F) the up projection;
  SwiGLU = silu(gate) * up with silu(g) = g / (1 + exp(-g)).
* Weights carry one fp32 scale per output channel; activations one fp32 scale per token (input)
  and per routed row (intermediate).
* Unused top-k slots (elastic k, k_t < k_max) hold expert id -1 and weight 0.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


# --------------------------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------------------------
def e4m3_table() -> np.ndarray:
    """float64 value of each of the 256 e4m3fn codes, from the bit-field definition."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        exp = (code >> 3) & 0xF
        man = code & 0x7
        if exp == 0xF and man == 0x7:
            vals[code] = np.nan
        elif exp == 0:
            vals[code] = sign * man * 2.0 ** -9          # subnormal: (m/8) * 2^(1-7)
        else:
            vals[code] = sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)
    return vals


E4M3_VALUES = e4m3_table()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(v) -> np.ndarray:
    """Round float64 values to e4m3fn codes: nearest, ties to even mantissa, saturate to +-448."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    nan = np.isnan(v)
    a = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))
    # exponent of the binade holding a: a in [2^(x-1), 2^x); below 2^-6 the quantum is fixed
    _, x = np.frexp(a)
    binade = np.maximum(x - 1, -6)
    quantum = np.ldexp(1.0, binade - 3)                 # 3 mantissa bits
    r = np.rint(a / quantum) * quantum                  # np.rint: round half to even
    r = np.minimum(r, E4M3_MAX)
    # back to bits
    _, xr = np.frexp(r)
    er = xr - 1
    normal = r >= 2.0 ** -6
    exp_field = np.where(normal, er + 7, 0)
    man_field = np.where(normal, r / np.ldexp(1.0, er) - 1.0, r / 2.0 ** -9)
    man_field = np.where(normal, man_field * 8.0, man_field)
    code = (exp_field.astype(np.int64) << 3) | np.rint(man_field).astype(np.int64)
    code = np.where(r == 0, 0, code)
    code = np.where(np.signbit(v), code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_round(v) -> np.ndarray:
    """One round-to-nearest-even rounding of float64 values to bf16; returns the uint16 bits."""
    v = np.asarray(v, dtype=np.float64)
    _, x = np.frexp(v)
    quantum = np.ldexp(1.0, np.maximum(x - 1, -126) - 7)   # 7 explicit mantissa bits
    r = np.rint(v / quantum) * quantum
    r32 = r.astype(np.float32)                              # exact: r has <= 8 significant bits
    return (r32.view(np.uint32) >> 16).astype(np.uint16)


# --------------------------------------------------------------------------------------------
# Steps of the layer
# --------------------------------------------------------------------------------------------
def router_logits(x: np.ndarray, router_w: np.ndarray, router_bias=None) -> np.ndarray:
    """l[t, e] = sum_d x[t, d] W[e, d] (+ b[e]), float64 (step 1)."""
    l = np.asarray(x, np.float64) @ np.asarray(router_w, np.float64).T
    if router_bias is not None:
        l = l + np.asarray(router_bias, np.float64)[None, :]
    return l


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over the expert axis (step 2, first half)."""
    z = np.exp(l - l.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def token_k(T: int, k: int, k_per_token=None) -> np.ndarray:
    if k_per_token is None:
        return np.full(T, int(k), dtype=np.int64)
    return np.asarray(k_per_token, dtype=np.int64)


def select_topk(l: np.ndarray, k_t: np.ndarray, k_max: int) -> np.ndarray:
    """ids[t, j]: the k_t largest logits in descending order, exact ties to the lower index.

    Slots j >= k_t hold -1 (step 2, selection).
    """
    T, E = l.shape
    ids = np.full((T, k_max), -1, dtype=np.int32)
    expert = np.broadcast_to(np.arange(E), l.shape)
    order = np.lexsort((expert, -l), axis=-1)           # primary key -l, then expert index
    for t in range(T):
        ids[t, :k_t[t]] = order[t, :k_t[t]]
    return ids


def routing_weights(l: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Softmax over all experts, then the selected probabilities renormalised to sum to 1."""
    p = softmax(l)
    w = np.zeros(ids.shape, dtype=np.float64)
    for t in range(ids.shape[0]):
        sel = ids[t][ids[t] >= 0]
        ps = p[t, sel]
        w[t, :len(sel)] = ps / ps.sum()
    return w


def quantize_rows_fp32(a) -> tuple:
    """Per-row dynamic FP8: s = fp32(amax) / 448 (1 if amax = 0), code = e4m3(fp32(a / s)).

    Both divisions are IEEE fp32 (numpy float32), the decision precision the kernels use.
    Returns (uint8 codes, float32 scales).
    """
    a = np.asarray(a, dtype=np.float32)
    amax = np.abs(a).max(axis=-1) if a.shape[-1] else np.zeros(a.shape[:-1], np.float32)
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    s = np.where(amax == 0, np.float32(1.0), s).astype(np.float32)
    q = (a / s[..., None]).astype(np.float32)
    return e4m3_encode(q.astype(np.float64)), s


def group_by_expert(ids: np.ndarray, k_t: np.ndarray, E: int):
    """Counting sort of the routed (token, slot) pairs by expert, token order kept (step 4).

    Returns counts [E], offsets [E+1] (exclusive prefix sum), perm_token [R] (token of each
    routed row, rows ordered by (expert, token)) and inv_row [T, k_max] (row of each (t, j),
    -1 for unused slots).
    """
    T, k_max = ids.shape
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k_t[t]):
            counts[ids[t, j]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    cursor = offsets[:-1].copy()
    perm_token = np.empty(int(offsets[-1]), dtype=np.int32)
    inv_row = np.full((T, k_max), -1, dtype=np.int32)
    for t in range(T):                       # ascending t: a stable order inside every group
        for j in range(k_t[t]):
            e = ids[t, j]
            r = cursor[e]
            perm_token[r] = t
            inv_row[t, j] = r
            cursor[e] += 1
    return counts.astype(np.int32), offsets.astype(np.int32), perm_token, inv_row


def silu(g: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def expert_ffn(xq, x_scale, w13, w13_scale, w2, w2_scale, return_intermediate=False):
    """FP8 SwiGLU expert on a block of rows of one expert (step 5).

    xq uint8 [n, d], x_scale fp32 [n]; w13 uint8 [2F, d], w13_scale fp32 [2F];
    w2 uint8 [d, F], w2_scale fp32 [d]. Returns o float64 [n, d].
      h   = x_scale[r] * w13_scale[j] * sum_d dq(xq[r, d]) dq(w13[j, d])    (exact products)
      act = silu(h[:, :F]) * h[:, F:]
      aq, s2 = per-row FP8 of act (fp32 decisions)
      o   = s2[r] * w2_scale[i] * sum_f dq(aq[r, f]) dq(w2[i, f])
    """
    F = w2.shape[1]
    X = e4m3_decode(xq)
    h = (X @ e4m3_decode(w13).T) * np.asarray(x_scale, np.float64)[:, None] \
        * np.asarray(w13_scale, np.float64)[None, :]
    act = silu(h[:, :F]) * h[:, F:]
    aq, s2 = quantize_rows_fp32(act.astype(np.float32))
    o = (e4m3_decode(aq) @ e4m3_decode(w2).T) * s2.astype(np.float64)[:, None] \
        * np.asarray(w2_scale, np.float64)[None, :]
    if return_intermediate:
        return o, dict(h=h, act=act, aq=aq, s2=s2)
    return o


def combine(o_rows, weights, inv_row, k_t, tokens, shared_out=None):
    """y[t] = sum_{j < k_t} w[t, j] o[inv_row[t, j]] (+ shared), float64, in token order (step 6).

    ``o_rows`` maps a routed row index to its float64 output vector; ``tokens`` lists the tokens
    to produce (all of them, or a sample).
    """
    d = next(iter(o_rows.values())).shape[0] if o_rows else (
        shared_out.shape[1] if shared_out is not None else 0)
    y = np.zeros((len(tokens), d), dtype=np.float64)
    for i, t in enumerate(tokens):
        for j in range(k_t[t]):
            y[i] += weights[t, j] * o_rows[int(inv_row[t, j])]
        if shared_out is not None:
            y[i] += shared_out[i]
    return y


# --------------------------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------------------------
def moe_forward(hidden_bits, router_w, router_bias, k, k_per_token, w13, w13_scale, w2,
                w2_scale, shared=None, tokens=None, k_max=None):
    """The layer's forward pass; every step above in order.

    hidden_bits uint16 [T, d] (bf16 bit patterns); router_w fp32 [E, d]; router_bias fp32 [E] or
    None; k int; k_per_token int32 [T] or None; w13 uint8 [E, 2F, d]; w13_scale fp32 [E, 2F];
    w2 uint8 [E, d, F]; w2_scale fp32 [E, d]; shared = (w13s, w13s_scale, w2s, w2s_scale) or
    None. ``tokens``: optional sorted sample of tokens whose outputs are computed (routing and
    grouping always cover every token). Returns a dict of every intermediate.
    """
    hidden_bits = np.asarray(hidden_bits, dtype=np.uint16)
    T, d = hidden_bits.shape
    E = router_w.shape[0]
    k_t = token_k(T, k, k_per_token)
    if k_max is None:
        k_max = int(k_t.max()) if T else int(k)
    x = bf16_bits_to_f64(hidden_bits)

    logits = router_logits(x, router_w, router_bias)
    ids = select_topk(logits, k_t, k_max)
    w = routing_weights(logits, ids)
    counts, offsets, perm_token, inv_row = group_by_expert(ids, k_t, E)
    xq, x_scale = quantize_rows_fp32(x.astype(np.float32))

    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    wanted = np.zeros(T, dtype=bool)
    wanted[tokens] = True
    o_rows = {}
    for e in range(E):
        rows = np.arange(offsets[e], offsets[e + 1])
        rows = rows[wanted[perm_token[rows]]]
        if len(rows) == 0:
            continue
        tok = perm_token[rows]
        o = expert_ffn(xq[tok], x_scale[tok], w13[e], w13_scale[e], w2[e], w2_scale[e])
        for r, orow in zip(rows, o):
            o_rows[int(r)] = orow
    shared_out = None
    if shared is not None:
        w13s, s13s, w2s, s2s = shared
        shared_out = expert_ffn(xq[tokens], x_scale[tokens], w13s, s13s, w2s, s2s)
    y64 = combine(o_rows, w, inv_row, k_t, tokens, shared_out)
    return dict(logits=logits, topk_ids=ids, topk_w=w, k_t=k_t, counts=counts,
                offsets=offsets, perm_token=perm_token, inv_row=inv_row, xq=xq,
                x_scale=x_scale, o_rows=o_rows, shared_out=shared_out, tokens=tokens,
                y64=y64, y_bf16=bf16_round(y64))


def near_tie_tokens(logits: np.ndarray, k_t: np.ndarray, gap: float = 1e-4) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest logits differ by less than ``gap``."""
    T, E = logits.shape
    s = -np.sort(-logits, axis=-1)
    out = []
    for t in range(T):
        kk = int(k_t[t])
        if 0 < kk < E and s[t, kk - 1] - s[t, kk] < gap:
            out.append(t)
    return np.asarray(out, dtype=np.int64)
