"""Float64 CPU oracle for Looped Latent Attention (LLA) decode.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` call
it.  It shares no code with the CUDA path: plain NumPy in float64, written from
the method's definition so that a reader can check each step against the pages.

Pages this follows (cited by page title and section):

* [CR]  "Looped Latent Attention: 跨循环 KV 压缩精读" (cc.laoqi.cc close reading of
        arXiv 2607.15456v2).  §二.1 symbol table, §二.2 eq. (4) and its worked
        example, §二.3 pre-RoPE compression, §二.4 SVD initialisation,
        §二.6 LLA-2D, §四.9 Table 5 (serving; the full-memory fast path),
        §四.10 Table 9 and Appendix J (eviction budgets; decoupled RoPE).
* [GS]  "Looped Latent Attention: Cross-Loop KV Compression for Looped
        Transformers" (gist.science explainer), "Technisches Resümee":
        "Kernmechanismus" (encode / loop-specific decode formulas, LLA-2D),
        "Zentrale Beiträge" (ratio formula), "Training und Initialisierung".
* [PN]  daiwk Q&A digest, entry on RoPE pairing for Llama-family models
        (split-half pairing), background for the RoPE layout reading.

Conventions (row vectors throughout, as on [GS] Kernmechanismus):
  per-head  x = [x_0; ...; x_{T-1}] in R^{T d}, loop-major, 0-based loops.
  LLA-2D    x = concat over (t, h, i) in R^{T H d}, loop-major then head.
  encode    c   = (x - mu) W_down,              W_down in R^{(T d) x r}
  decode    x^_t = c W_up,t^T + mu_t,           W_up,t in R^{d x r}
  RoPE      split-half: pair (i, i + d/2) rotated by angle pos * base^(-2i/d).

Where the pages are silent, the reading taken is stated next to the function
that takes it.
Every function here is pinned: the codec, bookkeeping, RoPE and decode by
``tests/test_oracle_pins.py``, eviction by ``tests/test_evict.py``, the
full-memory path by ``tests/test_full_memory.py`` and decoupled RoPE by
``tests/test_decoupled_rope.py`` (their CPU tests).
"""
from __future__ import annotations

from dataclasses import dataclass
from fractions import Fraction

import numpy as np

MODE_PER_HEAD = 0
MODE_2D = 1


@dataclass(frozen=True)
class Cfg:
    """Codec geometry.  [CR §二.1]: T loops, H heads, d_head, latent widths r_k, r_v."""

    T: int
    H: int
    d: int
    r_k: int
    r_v: int
    mode: int = MODE_PER_HEAD
    rope_base: float = 10000.0

    @property
    def width(self) -> int:
        """Width of the concatenated trajectory that one latent encodes."""
        return self.T * self.d if self.mode == MODE_PER_HEAD else self.T * self.H * self.d


# --------------------------------------------------------------------------
# bf16 rounding (the cache number format).  Round-to-nearest-even from float64.
# --------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even), return float64.

    bfloat16 = 1 sign, 8 exponent, 7 stored mantissa bits (8 significant bits).
    Normal numbers keep 8 significant bits; below 2^-126 the spacing is fixed at
    2^-133 (subnormals).  Values past the largest finite bf16 plus half an ulp
    become +-inf.  Rounding happens once, straight from float64.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    finite = np.isfinite(x)
    out[~finite] = x[~finite]
    xf = x[finite]
    m, e = np.frexp(xf)                       # xf = m * 2^e, 0.5 <= |m| < 1
    normal = e >= -125                        # |x| >= 2^-126
    q = np.where(normal, np.ldexp(np.rint(np.ldexp(m, 8)), e - 8),
                 np.ldexp(np.rint(np.ldexp(xf, 133)), -133))
    max_bf16 = np.ldexp(255.0, 127 - 7)       # (2 - 2^-7) * 2^127
    q = np.where(np.abs(q) > max_bf16, np.copysign(np.inf, xf), q)
    out[finite] = q
    return out


# --------------------------------------------------------------------------
# Bookkeeping: exact cache sizes and ratio  ([CR §二.2 eq. (4)], [GS Zentrale Beiträge])
# --------------------------------------------------------------------------

def teacher_scalars_per_token_layer(cfg: Cfg) -> int:
    """Uncompressed loop-indexed cache: K and V for every loop and head: 2 T H d."""
    return 2 * cfg.T * cfg.H * cfg.d


def lla_scalars_per_token_layer(cfg: Cfg) -> int:
    """LLA cache: (r_k + r_v) per head, H heads; LLA-2D stores r_k + r_v in total [CR §二.6]."""
    per = cfg.r_k + cfg.r_v
    return per * cfg.H if cfg.mode == MODE_PER_HEAD else per


def compression_ratio(cfg: Cfg) -> Fraction:
    """Exact ratio of persistent cache scalars at equal precision.

    Per head this is 2 T d_head / (r_k + r_v) ([GS Zentrale Beiträge], [CR eq. (4)]);
    for LLA-2D it is 2 T H d / (r_k + r_v).
    """
    return Fraction(teacher_scalars_per_token_layer(cfg), lla_scalars_per_token_layer(cfg))


def cache_bytes(cfg: Cfg, tokens: int, layers: int, bytes_per_scalar: int = 2) -> int:
    """Persistent latent-cache bytes for ``tokens`` tokens over ``layers`` shared layers."""
    return lla_scalars_per_token_layer(cfg) * tokens * layers * bytes_per_scalar


def teacher_cache_bytes(cfg: Cfg, tokens: int, layers: int, bytes_per_scalar: int = 2) -> int:
    return teacher_scalars_per_token_layer(cfg) * tokens * layers * bytes_per_scalar


# --------------------------------------------------------------------------
# Codec: encode / loop-specific decode ([GS Kernmechanismus], [CR §二.1])
# --------------------------------------------------------------------------

def encode(x: np.ndarray, mu: np.ndarray, W_down: np.ndarray) -> np.ndarray:
    """c = (x - mu) W_down.  x: [..., W] concatenated trajectory, mu: [W], W_down: [W, r]."""
    x = np.asarray(x, dtype=np.float64)
    return (x - np.asarray(mu, dtype=np.float64)) @ np.asarray(W_down, dtype=np.float64)


def reconstruct(c: np.ndarray, W_up_t: np.ndarray, mu_t: np.ndarray) -> np.ndarray:
    """x^_t = c W_up,t^T + mu_t.  c: [..., r], W_up_t: [d, r], mu_t: [d]."""
    c = np.asarray(c, dtype=np.float64)
    return c @ np.asarray(W_up_t, dtype=np.float64).T + np.asarray(mu_t, dtype=np.float64)


# --------------------------------------------------------------------------
# RoPE, split-half layout ([CR §二.3]: applied after reconstruction, full dimension)
# --------------------------------------------------------------------------

def rope_inv_freq(d: int, base: float) -> np.ndarray:
    """theta_i = base^(-2 i / d) for i < d/2, in float64."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate pair (x_i, x_{i+d/2}) by angle pos * theta_i.

    x: [..., d]; pos: integer array broadcastable to x.shape[:-1].
    Angles are formed in float64 (reading: the pages fix no RoPE precision).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(d, base)
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * cos - b * sin, a * sin + b * cos], axis=-1)


# --------------------------------------------------------------------------
# Attention for one query (decode) over a history plus the in-flight token
# --------------------------------------------------------------------------

def attention_plain(q, K_hist, V_hist, pos_hist, k_self, v_self, q_pos, base, scale=None):
    """Decode attention over an uncompressed per-loop cache.

    q, k_self, v_self: [d] pre-RoPE; K_hist, V_hist: [n, d] pre-RoPE; pos_hist: [n].
    Scores s = RoPE(q, q_pos) . RoPE(k, pos) * scale over the history and the
    in-flight token (at q_pos); softmax with max subtraction; output sum p v.
    Returns (out [d], p_hist [n], p_self).
    """
    q = np.asarray(q, np.float64)
    d = q.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    K_hist = np.asarray(K_hist, np.float64).reshape(-1, d)
    V_hist = np.asarray(V_hist, np.float64).reshape(-1, d)
    qr = rope(q, q_pos, base)
    kr = rope(K_hist, np.asarray(pos_hist), base)
    ks = rope(np.asarray(k_self, np.float64), q_pos, base)
    s = np.concatenate([kr @ qr, [ks @ qr]]) * scale
    s = s - s.max()
    p = np.exp(s)
    p = p / p.sum()
    out = p[:-1] @ V_hist + p[-1] * np.asarray(v_self, np.float64)
    return out, p[:-1], p[-1]


def decode_attention(q, k_self, v_self, c_k, c_v, W_up_k_t, W_up_v_t, mu_k_t, mu_v_t,
                     positions, q_pos, base, scale=None):
    """LLA decode attention at loop t, direct form.

    Rebuild loop t's history K and V from the latents ([GS Kernmechanismus]),
    then attend as ``attention_plain``.  The in-flight token's loop-t K/V is exact
    (it is encoded only after its last loop).  Returns out [d].
    """
    K = reconstruct(c_k, W_up_k_t, mu_k_t)
    V = reconstruct(c_v, W_up_v_t, mu_v_t)
    out, _, _ = attention_plain(q, K, V, positions, k_self, v_self, q_pos, base, scale)
    return out


def decode_attention_absorbed(q, k_self, v_self, c_k, c_v, W_up_k_t, W_up_v_t, mu_k_t, mu_v_t,
                              positions, q_pos, base, scale=None):
    """Same result with V never rebuilt per token.

    Because the weights p sum to one over history plus self,
      sum_j p_j (c_v,j W^T + mu) + p_self v_self
        = (sum_j p_j c_v,j) W^T + (sum_j p_j) mu + p_self v_self,
    so values are summed in latent space and up-projected once.
    """
    K = reconstruct(c_k, W_up_k_t, mu_k_t)
    d = np.asarray(q).shape[-1]
    zeros = np.zeros((K.shape[0], d))
    _, p_hist, p_self = attention_plain(q, K, zeros, positions, k_self, np.zeros(d), q_pos,
                                        base, scale)
    W_up_v_t = np.asarray(W_up_v_t, np.float64)
    c_v = np.asarray(c_v, np.float64).reshape(K.shape[0], W_up_v_t.shape[1])
    o_lat = p_hist @ c_v
    return (o_lat @ W_up_v_t.T
            + p_hist.sum() * np.asarray(mu_v_t, np.float64)
            + p_self * np.asarray(v_self, np.float64))


# --------------------------------------------------------------------------
# Whole-cache wrappers with the library's data layout (used by parity tests)
# --------------------------------------------------------------------------

@dataclass
class Codec:
    """fp64 codec parameters.

    per-head: W_down_[kv] [H, T*d, r], W_up_[kv] [H, T, d, r], mu_[kv] [H, T*d]
    LLA-2D:   W_down_[kv] [T*H*d, r],  W_up_[kv] [T, H, d, r], mu_[kv] [T*H*d]
    """

    W_down_k: np.ndarray
    W_down_v: np.ndarray
    W_up_k: np.ndarray
    W_up_v: np.ndarray
    mu_k: np.ndarray
    mu_v: np.ndarray


def w_up_t(cfg: Cfg, W_up: np.ndarray, t: int, h: int) -> np.ndarray:
    return W_up[h, t] if cfg.mode == MODE_PER_HEAD else W_up[t, h]


def mu_t(cfg: Cfg, mu: np.ndarray, t: int, h: int) -> np.ndarray:
    """Loop-t (and head-h) slice of the concatenated mean."""
    d = cfg.d
    if cfg.mode == MODE_PER_HEAD:
        return mu[h, t * d:(t + 1) * d]
    off = (t * cfg.H + h) * d
    return mu[off:off + d]


def encode_tokens(cfg: Cfg, codec: Codec, x_k, x_v):
    """Encode finished tokens.  x_[kv]: [N, T, H, d] (per-loop K/V rows of each token).

    Returns unrounded latents: per-head [N, H, r], LLA-2D [N, r].
    """
    x_k = np.asarray(x_k, np.float64)
    x_v = np.asarray(x_v, np.float64)
    N = x_k.shape[0]
    if cfg.mode == MODE_PER_HEAD:
        ck = np.empty((N, cfg.H, cfg.r_k))
        cv = np.empty((N, cfg.H, cfg.r_v))
        for h in range(cfg.H):
            xk = x_k[:, :, h, :].reshape(N, cfg.T * cfg.d)    # loop-major concat
            xv = x_v[:, :, h, :].reshape(N, cfg.T * cfg.d)
            ck[:, h] = encode(xk, codec.mu_k[h], codec.W_down_k[h])
            cv[:, h] = encode(xv, codec.mu_v[h], codec.W_down_v[h])
        return ck, cv
    xk = x_k.reshape(N, -1)                                     # (t, h, i) order
    xv = x_v.reshape(N, -1)
    return encode(xk, codec.mu_k, codec.W_down_k), encode(xv, codec.mu_v, codec.W_down_v)


def decode_attn_cache(cfg: Cfg, codec: Codec, t: int, q, k_self, v_self, c_k, c_v,
                      positions, q_pos, ctx_len, pairs=None, scale=None, absorbed=False):
    """Decode attention for a batch, library layout.

    q, k_self, v_self: [B, H, d]; c_k: per-head [B, n_cap, H, r_k], 2D [B, n_cap, r_k];
    positions: [B, n_cap]; q_pos, ctx_len: [B].  ``pairs`` restricts the work to a
    list of (b, h); the result holds NaN elsewhere.  Returns out [B, H, d].
    """
    q = np.asarray(q, np.float64)
    B, H, d = q.shape
    out = np.full((B, H, d), np.nan)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(H)]
    fn = decode_attention_absorbed if absorbed else decode_attention
    for b, h in pairs:
        n = int(ctx_len[b])
        if cfg.mode == MODE_PER_HEAD:
            ck = np.asarray(c_k[b, :n, h], np.float64)
            cv = np.asarray(c_v[b, :n, h], np.float64)
        else:
            ck = np.asarray(c_k[b, :n], np.float64)
            cv = np.asarray(c_v[b, :n], np.float64)
        out[b, h] = fn(q[b, h], k_self[b, h], v_self[b, h], ck, cv,
                       w_up_t(cfg, codec.W_up_k, t, h), w_up_t(cfg, codec.W_up_v, t, h),
                       mu_t(cfg, codec.mu_k, t, h), mu_t(cfg, codec.mu_v, t, h),
                       np.asarray(positions[b, :n]), int(q_pos[b]), cfg.rope_base, scale)
    return out


# --------------------------------------------------------------------------
# SVD initialisation ([CR §二.4], [GS Training und Initialisierung])
# --------------------------------------------------------------------------

def svd_init(X: np.ndarray, r: int):
    """Codec from calibration rows X [N, W] (concatenated trajectories).

    mu = column mean; W_down = top-r right singular vectors of X - mu, ordered by
    singular value.  Sign reading: each column's entry of largest magnitude is
    made positive (the pages fix no sign).  Returns (mu [W], W_down [W, r], sigma).
    """
    X = np.asarray(X, np.float64)
    mu = X.mean(axis=0)
    _, sigma, Vt = np.linalg.svd(X - mu, full_matrices=False)
    W = Vt[:r].T.copy()
    idx = np.argmax(np.abs(W), axis=0)
    sgn = np.sign(W[idx, np.arange(W.shape[1])])
    sgn[sgn == 0] = 1.0
    return mu, W * sgn, sigma


def loop_slices(W_down: np.ndarray, T: int, d: int, H: int | None = None) -> np.ndarray:
    """W_up,t initialised as the loop-t rows of W_down ([CR §二.4]).

    per-head: returns [T, d, r]; LLA-2D (H given): returns [T, H, d, r].
    """
    r = W_down.shape[1]
    if H is None:
        return W_down.reshape(T, d, r).copy()
    return W_down.reshape(T, H, d, r).copy()


def svd_codec(cfg: Cfg, calib_k: np.ndarray, calib_v: np.ndarray) -> Codec:
    """Build a full codec by SVD from calibration tokens calib_[kv]: [N, T, H, d]."""
    N = calib_k.shape[0]
    if cfg.mode == MODE_PER_HEAD:
        parts = {"k": ([], [], []), "v": ([], [], [])}
        for key, X, r in (("k", calib_k, cfg.r_k), ("v", calib_v, cfg.r_v)):
            for h in range(cfg.H):
                mu, Wd, _ = svd_init(X[:, :, h, :].reshape(N, cfg.T * cfg.d), r)
                parts[key][0].append(Wd)
                parts[key][1].append(loop_slices(Wd, cfg.T, cfg.d))
                parts[key][2].append(mu)
        return Codec(np.stack(parts["k"][0]), np.stack(parts["v"][0]),
                     np.stack(parts["k"][1]), np.stack(parts["v"][1]),
                     np.stack(parts["k"][2]), np.stack(parts["v"][2]))
    mk, Wk, _ = svd_init(calib_k.reshape(N, -1), cfg.r_k)
    mv, Wv, _ = svd_init(calib_v.reshape(N, -1), cfg.r_v)
    return Codec(Wk, Wv, loop_slices(Wk, cfg.T, cfg.d, cfg.H), loop_slices(Wv, cfg.T, cfg.d, cfg.H),
                 mk, mv)


# --------------------------------------------------------------------------
# Eviction composed with LLA ([CR] §四.10, Table 9 and Appendix J)
# --------------------------------------------------------------------------

def evict_keep(n: int, sink: int, window: int) -> np.ndarray:
    """History indices kept by a sink + window retention budget out of n tokens.

    [CR] §四.10 evaluates LLA under a 260-token budget, 4 sink tokens plus a
    256-token window, and Appendix J under a 1024-token one: the first ``sink``
    tokens and the ``window`` most recent ones stay.  Each keeps its own position
    (eviction drops tokens, it does not renumber the survivors; the page does not
    say, and this is the plain reading).
    """
    if n <= sink + window:
        return np.arange(n)
    return np.concatenate([np.arange(sink), np.arange(n - window, n)])


def decode_attention_evicted(q, k_self, v_self, c_k, c_v, W_up_k_t, W_up_v_t, mu_k_t, mu_v_t,
                             pos_hist, q_pos, base, sink, window, scale=None):
    """decode_attention over the tokens that sink + window keeps.

    c_k, c_v and pos_hist cover the whole history (n rows); the in-flight token
    is attended as always.
    """
    keep = evict_keep(len(pos_hist), sink, window)
    pos_hist = np.asarray(pos_hist)
    return decode_attention(q, k_self, v_self, np.asarray(c_k)[keep], np.asarray(c_v)[keep],
                            W_up_k_t, W_up_v_t, mu_k_t, mu_v_t, pos_hist[keep], q_pos, base,
                            scale)


# --------------------------------------------------------------------------
# Full-memory fast path ([CR] §四.9, Table 5 row "full-memory fast path" and the
# paragraph after the table; §二.3 for where RoPE sits)
# --------------------------------------------------------------------------

def full_memory_kv(c_k, c_v, W_up_k_t, W_up_v_t, mu_k_t, mu_v_t, positions, base,
                   round_bf16=True):
    """Loop-t K and V of a history as a full cache keeps them.

    [CR] §四.9: the full-memory fast path stores the complete rebuilt K/V (so it
    gives up the cache saving) instead of rebuilding on every read.  Per [CR]
    §二.3 the codec works on pre-RoPE K and the model rotates the rebuilt key at
    its position before caching it, so the stored key is
        K_j = RoPE(c_k,j W_up,k,t^T + mu_k,t, positions[j])
    and the stored value V_j = c_v,j W_up,v,t^T + mu_v,t.  The cache number
    format is bf16 (2 bytes per scalar, as in the Table 5 teacher row), so both
    are rounded once; ``round_bf16=False`` keeps float64.
    Returns (K [n, d], V [n, d]).
    """
    K = rope(reconstruct(c_k, W_up_k_t, mu_k_t), np.asarray(positions), base)
    V = reconstruct(c_v, W_up_v_t, mu_v_t)
    if round_bf16:
        return bf16_round(K), bf16_round(V)
    return K, V


def decode_attention_full(q, k_self, v_self, K_rot, V, q_pos, base, scale=None):
    """Ordinary decode attention over a full cache whose keys are already rotated.

    q, k_self, v_self: [d] pre-RoPE (the in-flight token, loop t); K_rot, V: [n, d].
      s_j    = scale * RoPE(q, q_pos) . K_rot,j
      s_self = scale * RoPE(q, q_pos) . RoPE(k_self, q_pos)
      p      = softmax over the n history scores and s_self
      out    = sum_j p_j V_j + p_self v_self
    """
    q = np.asarray(q, np.float64)
    d = q.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    K_rot = np.asarray(K_rot, np.float64).reshape(-1, d)
    V = np.asarray(V, np.float64).reshape(-1, d)
    q_rot = rope(q, q_pos, base)
    scores = np.empty(K_rot.shape[0] + 1)
    for j in range(K_rot.shape[0]):
        scores[j] = scale * float(np.dot(q_rot, K_rot[j]))
    scores[-1] = scale * float(np.dot(q_rot, rope(np.asarray(k_self, np.float64), q_pos, base)))
    w = np.exp(scores - scores.max())
    w /= w.sum()
    return w[:-1] @ V + w[-1] * np.asarray(v_self, np.float64)


def full_cache(cfg: Cfg, codec: Codec, t: int, c_k, c_v, positions, ctx_len, round_bf16=True):
    """The full-memory cache of loop t in the library's layout, head-major.

    c_k, c_v, positions: latent-cache layout ([B, n_cap, H, r] per head, [B, n_cap, r]
    LLA-2D; positions [B, n_cap]).  Returns (K [B, H, n_cap, d], V [B, H, n_cap, d])
    with rows j < ctx_len[b] filled by ``full_memory_kv`` and the rest zero.
    """
    B, n_cap = np.asarray(positions).shape
    K = np.zeros((B, cfg.H, n_cap, cfg.d))
    V = np.zeros((B, cfg.H, n_cap, cfg.d))
    for b in range(B):
        n = int(ctx_len[b])
        for h in range(cfg.H):
            if cfg.mode == MODE_PER_HEAD:
                ck, cv = np.asarray(c_k[b, :n, h]), np.asarray(c_v[b, :n, h])
            else:
                ck, cv = np.asarray(c_k[b, :n]), np.asarray(c_v[b, :n])
            K[b, h, :n], V[b, h, :n] = full_memory_kv(
                ck, cv, w_up_t(cfg, codec.W_up_k, t, h), w_up_t(cfg, codec.W_up_v, t, h),
                mu_t(cfg, codec.mu_k, t, h), mu_t(cfg, codec.mu_v, t, h),
                np.asarray(positions[b, :n]), cfg.rope_base, round_bf16)
    return K, V


def decode_attn_full_cache(cfg: Cfg, q, k_self, v_self, K_full, V_full, q_pos, ctx_len,
                           scale=None):
    """``decode_attention_full`` for a batch.  q, k_self, v_self: [B, H, d];
    K_full, V_full: [B, H, n_cap, d]; q_pos, ctx_len: [B].  Returns [B, H, d]."""
    q = np.asarray(q, np.float64)
    B, H, d = q.shape
    out = np.zeros((B, H, d))
    for b in range(B):
        n = int(ctx_len[b])
        for h in range(H):
            out[b, h] = decode_attention_full(q[b, h], k_self[b, h], v_self[b, h],
                                              K_full[b, h, :n], V_full[b, h, :n],
                                              int(q_pos[b]), cfg.rope_base, scale)
    return out


# --------------------------------------------------------------------------
# Decoupled RoPE ([CR] §四.10, Appendix J and Tables 13-14): a NoPE content path
# absorbed into the query plus an explicit rotary branch of d_rope dims
# --------------------------------------------------------------------------

def rope_partial(x, pos, base: float, d_rope: int) -> np.ndarray:
    """RoPE on the first d_rope dims of x only, as a rotary vector of its own width
    (split-half pairs (i, i + d_rope/2) at angle pos * base^(-2i/d_rope)); the other
    d - d_rope dims pass through unrotated.  d_rope = d is the full RoPE of ``rope``.

    Reading: [CR] App. J names a NoPE content path and an explicit rotary branch of
    d_rope = 64 or 32 dims without saying which dims rotate; the plain reading is
    the usual partial-rotary layout (leading dims, their own frequency ladder).
    """
    x = np.asarray(x, np.float64)
    if d_rope == 0:
        return x.copy()
    return np.concatenate([rope(x[..., :d_rope], pos, base), x[..., d_rope:]], axis=-1)


def decode_attention_decoupled(q, k_self, v_self, c_k, c_v, W_up_k_t, W_up_v_t, mu_k_t, mu_v_t,
                               positions, q_pos, base, d_rope, scale=None):
    """Decode attention with decoupled RoPE, direct form: rebuild K and V from the
    latents, rotate the first d_rope dims of every key at its position and of the
    query (and the in-flight key) at q_pos, attend.  Returns out [d]."""
    q = np.asarray(q, np.float64)
    d = q.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    K = reconstruct(c_k, W_up_k_t, mu_k_t).reshape(-1, d)
    V = reconstruct(c_v, W_up_v_t, mu_v_t).reshape(-1, d)
    qr = rope_partial(q, q_pos, base, d_rope)
    Kr = rope_partial(K, np.asarray(positions), base, d_rope)
    ks = rope_partial(k_self, q_pos, base, d_rope)
    s = np.concatenate([Kr @ qr, [ks @ qr]]) * scale
    p = np.exp(s - s.max())
    p /= p.sum()
    return p[:-1] @ V + p[-1] * np.asarray(v_self, np.float64)


def decode_attention_decoupled_absorbed(q, k_self, v_self, c_k, c_v, W_up_k_t, W_up_v_t, mu_k_t,
                                        mu_v_t, positions, q_pos, base, d_rope, scale=None):
    """The same result computed the way App. J describes it: the NoPE content score
    is taken in latent space with the query absorbed into the up-projection,
        q_nope . (c W_nope^T + mu_nope) = (W_nope^T q_nope) . c + q_nope . mu_nope,
    only the d_rope rotary dims of each key are rebuilt and rotated, and values
    are summed in latent space and up-projected once."""
    q = np.asarray(q, np.float64)
    d = q.shape[-1]
    scale = 1.0 / np.sqrt(d) if scale is None else float(scale)
    Wk = np.asarray(W_up_k_t, np.float64)
    mk = np.asarray(mu_k_t, np.float64)
    c_k = np.asarray(c_k, np.float64).reshape(-1, Wk.shape[1])
    q_nope = q[d_rope:]
    a_nope = Wk[d_rope:].T @ q_nope                    # absorbed query, [r_k]
    s_hist = c_k @ a_nope + q_nope @ mk[d_rope:]
    if d_rope:
        K_rope = c_k @ Wk[:d_rope].T + mk[:d_rope]     # explicit rotary branch only
        q_rope = rope(q[:d_rope], q_pos, base)
        s_hist = s_hist + rope(K_rope, np.asarray(positions), base) @ q_rope
    ks = np.asarray(k_self, np.float64)
    s_self = float(rope_partial(ks, q_pos, base, d_rope) @ rope_partial(q, q_pos, base, d_rope))
    s = np.concatenate([s_hist, [s_self]]) * scale
    p = np.exp(s - s.max())
    p /= p.sum()
    Wv = np.asarray(W_up_v_t, np.float64)
    c_v = np.asarray(c_v, np.float64).reshape(-1, Wv.shape[1])
    o_lat = p[:-1] @ c_v
    return (o_lat @ Wv.T + p[:-1].sum() * np.asarray(mu_v_t, np.float64)
            + p[-1] * np.asarray(v_self, np.float64))


def decode_attn_cache_decoupled(cfg: Cfg, codec: Codec, t: int, q, k_self, v_self, c_k, c_v,
                                positions, q_pos, ctx_len, d_rope, pairs=None, scale=None):
    """``decode_attention_decoupled`` for a batch in the library's layout (see
    ``decode_attn_cache``).  Returns out [B, H, d] (NaN outside ``pairs``)."""
    q = np.asarray(q, np.float64)
    B, H, d = q.shape
    out = np.full((B, H, d), np.nan)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        n = int(ctx_len[b])
        if cfg.mode == MODE_PER_HEAD:
            ck, cv = np.asarray(c_k[b, :n, h]), np.asarray(c_v[b, :n, h])
        else:
            ck, cv = np.asarray(c_k[b, :n]), np.asarray(c_v[b, :n])
        out[b, h] = decode_attention_decoupled(
            q[b, h], k_self[b, h], v_self[b, h], ck, cv, w_up_t(cfg, codec.W_up_k, t, h),
            w_up_t(cfg, codec.W_up_v, t, h), mu_t(cfg, codec.mu_k, t, h),
            mu_t(cfg, codec.mu_v, t, h), np.asarray(positions[b, :n]), int(q_pos[b]),
            cfg.rope_base, d_rope, scale)
    return out
