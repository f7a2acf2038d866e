"""fp64 CPU oracle of the latent mixture-of-experts FFN block.

TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU-baseline
leg of the benchmark may import this module.  It is plain numpy in float64,
slow on purpose, and shares no code with the CUDA path: every storage format
is decoded here from its definition, every step follows the method as the
pages state it, and no blocking or fusion is done beyond what the definition
states.  A matrix product (numpy ``@``) is used as a step.

What the block computes (the teardown article "Edge0-145B: a Qwen MoE with its
experts squeezed, and a 51B table left on the SSD", section "A latent in
front of the experts", layer equation; the Edge0 145B / 120B model page,
"Model profile" and the architecture tables):

    y = U_g( sum_{e in top-10} w_e E_e(D_g x) ) + shared(x)

read per group: every expert carries one of 8 group labels; a token is
compressed by D_g of each group g that one of its ten experts belongs to,
the experts of group g run on D_g x, their routing-weighted outputs are
summed per group and widened back by U_g, and the shared expert runs on x
at full width.  The router (softmax over all experts, top-10, renormalise,
lowest index wins ties, bias added to the logits) is not printed on the
pages; it is taken from the task's workload statement.

Parity pins: tests/test_oracle_pins.py checks every function here against
values the pages print (byte totals of the formats), library conversions
(fp8/bf16 dtypes), closed forms, special cases and brute force.
"""
from __future__ import annotations

import numpy as np

Q8_0 = 8
Q4_0 = 4

# ----------------------------------------------------------------------------
# scalar storage formats
# ----------------------------------------------------------------------------


def bf16_to_f64(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (the high half of an IEEE binary32)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def fp16_to_f64(bits) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64 (sign, 5-bit exponent bias 15, 10-bit fraction)."""
    u = np.asarray(bits, dtype=np.int64) & 0xFFFF
    s = u >> 15
    e = (u >> 10) & 0x1F
    f = u & 0x3FF
    mag = np.where(e == 0, f * 2.0 ** -24, (1.0 + f / 1024.0) * np.exp2(e.astype(np.float64) - 15.0))
    mag = np.where(e == 31, np.where(f == 0, np.inf, np.nan), mag)
    return np.where(s == 1, -mag, mag)


def e2m1_to_f64(code) -> np.ndarray:
    """FP4 E2M1 code (4 bits: sign, 2-bit exponent bias 1, 1-bit mantissa) -> float64.

    Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (OCP Microscaling formats, E2M1)."""
    c = np.asarray(code, dtype=np.int64) & 0xF
    s, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e.astype(np.float64) - 1.0))
    return np.where(s == 1, -mag, mag)


def e4m3fn_to_f64(code) -> np.ndarray:
    """FP8 E4M3 (fn: no infinities; S.1111.111 is NaN) -> float64.

    sign, 4-bit exponent bias 7, 3-bit mantissa; exponent 0 is subnormal
    (m/8 * 2^-6); the NVFP4 block scale of the teardown article ("What is
    4-bit": E4M3 scale per 16 values)."""
    c = np.asarray(code, dtype=np.int64) & 0xFF
    s, e, m = c >> 7, (c >> 3) & 0xF, c & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


# ----------------------------------------------------------------------------
# matrix storage formats (layouts documented in the header of the C-ABI)
# ----------------------------------------------------------------------------


def du_matrix_bytes(fmt: int, rows: int, cols: int) -> int:
    """Q8_0 stores 32 int8 + one fp16 scale per 32 weights (34 B); Q4_0 stores
    32 nibbles + one fp16 scale (18 B)."""
    return rows * cols // 32 * (34 if fmt == Q8_0 else 18)


def nvfp4_matrix_bytes(rows: int, cols: int) -> int:
    """E2M1 nibbles plus one E4M3 scale per 16 weights."""
    return rows * cols // 2 + rows * cols // 16


def expert_record_bytes(latent: int, ffn: int, expert_fmt: str = "nvfp4") -> int:
    """gate [ffn, latent], up [ffn, latent], down [latent, ffn] in NVFP4 plus a
    16-byte tail holding the three fp32 tensor scales (teardown article, "What
    is 4-bit": 1,935,376 B for 3,440,640 weights at latent 1792); or the Q3_K
    build: Q3_K gate and up, IQ4_NL down, no tail (1,630,720 B)."""
    if expert_fmt == "q3k":
        return 2 * (ffn * latent // 256 * 110) + latent * ffn // 32 * 18
    return 3 * nvfp4_matrix_bytes(ffn, latent) + 16


def decode_q8_0(blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Q8_0 matrix [rows, cols]: int8 q [cols/32][rows][32], then fp16 d [cols/32][rows];
    weight = d * q, blocks of 32 along cols."""
    nb = cols // 32
    q = np.frombuffer(blob, dtype=np.int8, count=rows * cols).reshape(nb, rows, 32).astype(np.float64)
    dbits = np.frombuffer(blob, dtype=np.uint16, count=nb * rows, offset=rows * cols).reshape(nb, rows)
    d = fp16_to_f64(dbits)
    w = q * d[:, :, None]                       # [nb, rows, 32]
    return w.transpose(1, 0, 2).reshape(rows, cols)


def decode_q4_0(blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Q4_0 matrix [rows, cols]: 16 bytes per block of 32, [cols/32][rows][16];
    byte j holds element j (low nibble) and element j+16 (high nibble);
    weight = d * (q - 8); then fp16 d [cols/32][rows]."""
    nb = cols // 32
    b = np.frombuffer(blob, dtype=np.uint8, count=rows * cols // 2).reshape(nb, rows, 16).astype(np.int64)
    q = np.concatenate([b & 0xF, b >> 4], axis=2).astype(np.float64)   # elements 0..15 then 16..31
    dbits = np.frombuffer(blob, dtype=np.uint16, count=nb * rows, offset=rows * cols // 2).reshape(nb, rows)
    d = fp16_to_f64(dbits)
    w = (q - 8.0) * d[:, :, None]
    return w.transpose(1, 0, 2).reshape(rows, cols)


def decode_du(fmt: int, blob: np.ndarray, rows: int, cols: int) -> np.ndarray:
    if fmt == Q8_0:
        return decode_q8_0(blob, rows, cols)
    if fmt == Q4_0:
        return decode_q4_0(blob, rows, cols)
    raise ValueError(f"unknown D/U format {fmt}")


def decode_nvfp4(qbytes: np.ndarray, sbytes: np.ndarray, ts: float, rows: int, cols: int) -> np.ndarray:
    """NVFP4 matrix [rows, cols]: codes [cols/32][rows][16 bytes] with element 2i
    in the low nibble of byte i and 2i+1 in the high nibble; E4M3 scales
    [cols/64][rows][4] with byte j scaling elements 16j..16j+15 of the group;
    weight = e2m1(code) * e4m3(scale) * ts (fp32 tensor scale)."""
    nb = cols // 32
    b = np.asarray(qbytes, dtype=np.uint8)[: rows * cols // 2].reshape(nb, rows, 16).astype(np.int64)
    codes = np.stack([b & 0xF, b >> 4], axis=3).reshape(nb, rows, 32)     # interleave lo, hi
    vals = e2m1_to_f64(codes).transpose(1, 0, 2).reshape(rows, cols)
    sc = np.asarray(sbytes, dtype=np.uint8)[: rows * cols // 16].reshape(cols // 64, rows, 4)
    scale = e4m3fn_to_f64(sc).transpose(1, 0, 2).reshape(rows, cols // 16)
    return vals * np.repeat(scale, 16, axis=1) * float(ts)


# The other expert build (model page, "Model profile": Q3_K gate/up, IQ4_NL
# down; teardown article, "What is 4-bit": 985,600 + 645,120 bytes per record
# at latent 1792).  The pages give names and byte counts; the arrangement is
# the one documented with the C ABI (planes over 128-column halves for Q3_K,
# Q4_0-like planes for IQ4_NL).

def iq4nl_levels() -> np.ndarray:
    """The 16 IQ4_NL levels as read here: standard normal quantiles at
    (i + 1/2) / 16, scaled so that the outermost is 127, rounded."""
    from statistics import NormalDist
    z = [NormalDist().inv_cdf((i + 0.5) / 16.0) for i in range(16)]
    return np.rint(127.0 * np.array(z) / z[-1])


def q3k_matrix_bytes(rows: int, cols: int) -> int:
    return rows * cols // 256 * 110


def iq4nl_matrix_bytes(rows: int, cols: int) -> int:
    return rows * cols // 32 * 18


def decode_q3k(blob, rows: int, cols: int) -> np.ndarray:
    """Q3_K matrix [rows, cols]: w = d * (sc_j - 32) * (q - 4)."""
    R, C = rows, cols
    nh = C // 128
    b = np.asarray(blob, np.uint8)
    lo = b[: nh * R * 32].reshape(nh, R, 32).astype(np.int64)
    hi = b[nh * R * 32: nh * R * 48].reshape(nh, R, 16).astype(np.int64)
    sc = b[nh * R * 48: nh * R * 54].reshape(nh, R, 6).astype(np.int64)
    d = fp16_to_f64(np.frombuffer(b[nh * R * 54: nh * R * 54 + 2 * (C // 256) * R].tobytes(), np.uint16)
                    .reshape(C // 256, R))
    e = np.arange(128)
    q_lo = (lo[:, :, 4 * (e // 16) + e % 4] >> (2 * ((e % 16) // 4))) & 3           # [nh, R, 128]
    q_hi = (hi[:, :, 4 * (e // 32) + e % 4] >> ((e % 32) // 4)) & 1
    q = q_lo | (q_hi << 2)
    word = sum(sc[:, :, k] << (8 * k) for k in range(6))                            # 48-bit words [nh, R]
    j = e // 16
    scj = (word[:, :, None] >> (6 * j)[None, None, :]) & 63                        # [nh, R, 128]
    dv = np.repeat(d, 2, axis=0)[:, :, None]                                       # d of each half
    w = dv * (scj - 32) * (q - 4)
    return w.transpose(1, 0, 2).reshape(R, C)


def decode_iq4nl(blob, rows: int, cols: int) -> np.ndarray:
    """IQ4_NL matrix [rows, cols]: w = d * level[q], q as in Q4_0."""
    nb = cols // 32
    b = np.asarray(blob, np.uint8)[: rows * cols // 2].reshape(nb, rows, 16).astype(np.int64)
    q = np.concatenate([b & 0xF, b >> 4], axis=2)
    dbits = np.frombuffer(np.asarray(blob, np.uint8)[rows * cols // 2: rows * cols // 2 + 2 * nb * rows].tobytes(),
                          np.uint16).reshape(nb, rows)
    w = iq4nl_levels()[q] * fp16_to_f64(dbits)[:, :, None]
    return w.transpose(1, 0, 2).reshape(rows, cols)


def decode_expert(record: np.ndarray, latent: int, ffn: int, expert_fmt: str = "nvfp4"):
    if expert_fmt == "q3k":
        rec = np.asarray(record, np.uint8)
        gb = q3k_matrix_bytes(ffn, latent)
        return (decode_q3k(rec[:gb], ffn, latent), decode_q3k(rec[gb:2 * gb], ffn, latent),
                decode_iq4nl(rec[2 * gb:2 * gb + iq4nl_matrix_bytes(latent, ffn)], latent, ffn))
    return _decode_expert_nvfp4(record, latent, ffn)


def _decode_expert_nvfp4(record: np.ndarray, latent: int, ffn: int):
    """-> (W_gate [ffn, latent], W_up [ffn, latent], W_down [latent, ffn]) in fp64."""
    nq = latent * ffn // 2
    ns = latent * ffn // 16
    rec = np.asarray(record, dtype=np.uint8)
    ts = np.frombuffer(rec[3 * nq + 3 * ns: 3 * nq + 3 * ns + 12].tobytes(), dtype=np.float32).astype(np.float64)
    shapes = [(ffn, latent), (ffn, latent), (latent, ffn)]
    mats = []
    for m, (r, c) in enumerate(shapes):
        mats.append(decode_nvfp4(rec[m * nq:(m + 1) * nq], rec[3 * nq + m * ns: 3 * nq + (m + 1) * ns], ts[m], r, c))
    return tuple(mats)


def expert_slice(experts: np.ndarray, e: int, latent: int, ffn: int, expert_fmt: str = "nvfp4") -> np.ndarray:
    rb = expert_record_bytes(latent, ffn, expert_fmt)
    return experts[e * rb:(e + 1) * rb]


def du_slice(blob: np.ndarray, fmt: int, g: int, rows: int, cols: int) -> np.ndarray:
    mb = du_matrix_bytes(fmt, rows, cols)
    return blob[g * mb:(g + 1) * mb]


# ----------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------


def route(x: np.ndarray, Wr: np.ndarray, b: np.ndarray | None, top_k: int):
    """Router over all experts.

    logits l = x W_r^T + b (the bias is added to the logits and so moves both
    the selection and the weights); experts are ordered by (logit descending,
    index ascending) and the first top_k kept; p = softmax(l) over all
    experts; w_k = p_k / sum of the kept p.  Returns (idx [T, K] int64,
    w [T, K] fp64, gap [T] = l_(K) - l_(K+1), logits [T, E])."""
    x = np.asarray(x, np.float64)
    logits = x @ np.asarray(Wr, np.float64).T
    if b is not None:
        logits = logits + np.asarray(b, np.float64)[None, :]
    T, E = logits.shape
    idx = np.zeros((T, top_k), np.int64)
    w = np.zeros((T, top_k), np.float64)
    gap = np.full(T, np.inf)
    for t in range(T):
        lt = logits[t]
        order = np.lexsort((np.arange(E), -lt))        # last key is primary: logit desc, then index asc
        sel = order[:top_k]
        p = np.exp(lt - lt.max())
        p = p / p.sum()
        idx[t] = sel
        w[t] = p[sel] / p[sel].sum()
        if top_k < E:
            gap[t] = lt[order[top_k - 1]] - lt[order[top_k]]
    return idx, w, gap, logits


# ----------------------------------------------------------------------------
# block
# ----------------------------------------------------------------------------


def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def shared_expert(x: np.ndarray, Wsg: np.ndarray, Wsu: np.ndarray, Wsd: np.ndarray) -> np.ndarray:
    """SwiGLU at full width: W_down (silu(W_gate x) * (W_up x)); x [T, H] -> [T, H]."""
    a = x @ Wsg.T
    u = x @ Wsu.T
    return (silu(a) * u) @ Wsd.T


def expert_apply(Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray, h: np.ndarray, act: str = "fp16") -> np.ndarray:
    """E_e : R^l -> R^F -> R^l, SwiGLU: W_down (silu(W_gate h) * (W_up h)).
    act = "nvfp4": h and z enter as their NVFP4 activation values (W4A4)."""
    if act == "nvfp4":
        h = nvfp4_act(h)
    a = Wg @ h
    u = Wu @ h
    z = silu(a) * u
    if act == "nvfp4":
        z = nvfp4_act(z)
    return Wd @ z


# ---- NVFP4 activations (the W4A4 mode) -------------------------------------
# The teardown article ("What is 4-bit") gives NVFP4 for the weights; the
# W4A4 mode applies it to the experts' inputs with the rule the pages leave
# open read plainly: one fp32 scale per row G = max|v| / (6 * 448), per 16
# elements the smallest E4M3 value s >= max|v_block| / (6 G), E2M1 codes
# nearest (ties to even, saturating) to v / (s G).  The decisions are taken
# in fp32 on the fp16-rounded row, as the kernels take them.

def _e4m3_positive() -> np.ndarray:
    return e4m3fn_to_f64(np.arange(0x7F))          # codes 0 .. 0x7E by value, 0x7F is NaN


def _e2m1_nearest(v: np.ndarray) -> np.ndarray:
    """Value of the E2M1 code nearest to each float32 v (ties to the even code, +-6 at most)."""
    mags = e2m1_to_f64(np.arange(8))
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[..., None] - mags)
    dmin = d.min(-1, keepdims=True)
    cand = d == dmin
    even = cand & (np.arange(8) % 2 == 0)
    code = np.where(even.any(-1), np.argmax(even, -1), np.argmax(cand, -1))
    return np.where(v < 0, -mags[code], mags[code])


def nvfp4_act(v: np.ndarray) -> np.ndarray:
    """NVFP4 activation values of one row v [K] (K % 16 == 0), fp64 out."""
    r = fp16_round(np.asarray(v, np.float64)).astype(np.float32)
    amax = np.float32(np.abs(r).max())
    G = np.float32(amax * np.float32(1.0 / 2688.0)) if amax > 0 else np.float32(1.0)
    e4 = _e4m3_positive()
    blocks = r.reshape(-1, 16)
    bmax = np.abs(blocks).max(1)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = (bmax / np.float32(np.float32(6.0) * G)).astype(np.float32)
    code = np.minimum(np.searchsorted(e4.astype(np.float32), s, side="left"), 0x7E)
    code = np.where(bmax > 0, np.maximum(code, 1), 0)
    sval = e4[code].astype(np.float32)
    sd = (sval * G).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = np.where(sd > 0, np.float32(1.0) / sd, np.float32(0.0)).astype(np.float32)
    q = _e2m1_nearest((blocks * inv[:, None]).astype(np.float32))
    out = q * e4[code][:, None] * np.float64(G)
    return np.where(bmax[:, None] > 0, out, 0.0).reshape(-1)


def fp16_round(v: np.ndarray) -> np.ndarray:
    """Nearest binary16 values (ties to even), as fp64."""
    return np.asarray(v, np.float64).astype(np.float16).astype(np.float64)


class Weights:
    """Decoded view of one layer's weights.  D_g, U_g and experts are decoded
    lazily and kept (a bounded number of experts at a time)."""

    def __init__(self, shape, layer: dict, max_cached_experts: int = 64):
        self.s = shape
        self.layer = layer
        H, L, Fs = shape.hidden, shape.latent, shape.shared_ffn
        rw = layer["router_w"]
        self.Wr = bf16_to_f64(rw) if rw.dtype == np.uint16 else np.asarray(rw, np.float64)
        self.b = None if layer.get("router_b") is None else np.asarray(layer["router_b"], np.float64)
        self.group = np.asarray(layer["expert_group"], np.int64)
        self.Wsg = bf16_to_f64(layer["shared_gate"]).reshape(Fs, H)
        self.Wsu = bf16_to_f64(layer["shared_up"]).reshape(Fs, H)
        self.Wsd = bf16_to_f64(layer["shared_down"]).reshape(H, Fs)
        self._D, self._U, self._E = {}, {}, {}
        self._max = max_cached_experts

    def D(self, g: int) -> np.ndarray:
        if g not in self._D:
            s = self.s
            self._D[g] = decode_du(s.du_fmt, du_slice(self.layer["D"], s.du_fmt, g, s.latent, s.hidden), s.latent, s.hidden)
        return self._D[g]

    def U(self, g: int) -> np.ndarray:
        if g not in self._U:
            s = self.s
            self._U[g] = decode_du(s.du_fmt, du_slice(self.layer["U"], s.du_fmt, g, s.hidden, s.latent), s.hidden, s.latent)
        return self._U[g]

    def expert(self, e: int):
        if e not in self._E:
            if len(self._E) >= self._max:
                self._E.pop(next(iter(self._E)))
            s = self.s
            f = getattr(s, "expert_fmt", "nvfp4")
            self._E[e] = decode_expert(expert_slice(self.layer["experts"], e, s.latent, s.ffn, f), s.latent, s.ffn, f)
        return self._E[e]


def latent_moe_forward(shape, layer: dict, x_bits: np.ndarray, residual_bits: np.ndarray | None = None,
                       inject_idx: np.ndarray | None = None, inject_w: np.ndarray | None = None,
                       weights: Weights | None = None, x_f64: np.ndarray | None = None):
    """One latent-MoE FFN block on tokens x [T, H] (bf16 bits, or fp64 via x_f64).

    Steps: route; for each token the set of hit groups G_t = {group(e_k)};
    h_{t,g} = D_g x_t for g in G_t; o_k = E_{e_k}(h_{t, group(e_k)});
    s_{t,g} = sum_{k: group(e_k) = g} w_k o_k;
    y_t = sum_{g in G_t} U_g s_{t,g} + shared(x_t) (+ residual_t).

    inject_idx / inject_w replace the router's choice (used where the top-K
    boundary is closer than the comparison can resolve).  Returns
    (y [T, H] fp64, idx, w, gap)."""
    W = weights if weights is not None else Weights(shape, layer)
    x = bf16_to_f64(x_bits) if x_f64 is None else np.asarray(x_f64, np.float64)
    T = x.shape[0]
    idx, w, gap, _ = route(x, W.Wr, W.b, shape.top_k)
    if inject_idx is not None:
        idx = np.asarray(inject_idx, np.int64)
        w = np.asarray(inject_w, np.float64)
    y = shared_expert(x, W.Wsg, W.Wsu, W.Wsd)
    # expert outputs o[t, k]; each (t, k) pair is computed alone, the decoded
    # weights of an expert are reused by every pair routed to it
    o = np.zeros((T, shape.top_k, shape.latent))
    pairs = {}
    for t in range(T):
        for k in range(shape.top_k):
            pairs.setdefault(int(idx[t, k]), []).append((t, k))
    h_cache = {}
    for e in sorted(pairs):
        g = int(W.group[e])
        Wg, Wu, Wd = W.expert(e)
        for (t, k) in pairs[e]:
            if (t, g) not in h_cache:
                h_cache[(t, g)] = W.D(g) @ x[t]
            o[t, k] = expert_apply(Wg, Wu, Wd, h_cache[(t, g)], getattr(shape, "act_fmt", "fp16"))
    for t in range(T):
        hit = sorted({int(W.group[e]) for e in idx[t]})
        for g in hit:
            s_tg = np.zeros(shape.latent)
            for k in range(shape.top_k):
                if int(W.group[idx[t, k]]) == g:
                    s_tg += w[t, k] * o[t, k]
            y[t] += W.U(g) @ s_tg
    if residual_bits is not None:
        y = y + bf16_to_f64(residual_bits)
    return y, idx, w, gap


def rmsnorm(v: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """gamma * v / sqrt(mean(v^2) + eps), per row."""
    v = np.asarray(v, np.float64)
    return np.asarray(gamma, np.float64)[None, :] * v / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + eps)


def stack_layer_forward(shape, layer: dict, x_bits: np.ndarray, gamma: np.ndarray, eps: float,
                        weights: Weights | None = None, inject_idx=None, inject_w=None):
    """One pre-norm residual layer of the stack: x + block(RMSNorm(x)).
    x is the layer input as bf16 bits (the stack keeps its residual stream in
    bf16).  Returns (y fp64, idx, w, gap)."""
    x = bf16_to_f64(x_bits)
    xn = rmsnorm(x, gamma, eps)
    y, idx, w, gap = latent_moe_forward(shape, layer, None, inject_idx=inject_idx, inject_w=inject_w,
                                        weights=weights, x_f64=xn)
    return x + y, idx, w, gap


def rel_l2(a: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(np.asarray(a, np.float64) - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs_over_rms(a: np.ndarray, ref: np.ndarray) -> float:
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(np.asarray(a, np.float64) - ref)) / max(rms, 1e-300))
