/*
 * lla.h -- C ABI of the Looped Latent Attention (LLA) decode library for NVIDIA
 * B200 (sm_100a).
 *
 * What the method computes (pages cited by title and section):
 *   "Looped Latent Attention: Cross-Loop KV Compression for Looped Transformers"
 *   (gist.science explainer), Technisches Resümee / Kernmechanismus:
 *     encode                c    = (x - mu) W_down
 *     loop-specific decode  x^_t = c W_up,t^T + mu_t
 *   where x = [x_1; ...; x_T] is one token's pre-RoPE K (or V) for every loop.
 *   "Looped Latent Attention: 跨循环 KV 压缩精读" (cc.laoqi.cc close reading),
 *   §二.1 symbol table (W_down is (T d_head) x r, W_up,t is d_head x r),
 *   §二.2 eq. (4) (exact ratio 2 T d_head / (r_k + r_v)), §二.3 (compress before
 *   RoPE, rotate the rebuilt K at its position), §二.6 (LLA-2D folds the heads
 *   into one latent of input width T H d_head; the latent-store path keeps only
 *   latents and rebuilds on read).
 *
 * Conventions
 *   - Loops are 0-based (t = 0 .. T-1); the pages count from 1.
 *   - Row vectors, as on the pages.  Every matrix is row-major, C order.
 *   - bf16 values are passed as their uint16_t bit patterns.
 *   - RoPE is the split-half layout: pair (i, i + d/2) rotates by angle
 *     pos * rope_base^(-2 i / d).  Scores are scaled by sm_scale (1/sqrt(d) when 0).
 *   - The in-flight token (the one whose loops are still running) is not in the
 *     latent cache: its loop-t K and V are passed exactly (k_self, v_self) and it
 *     attends to itself at q_pos.  It is encoded with lla_encode after its last loop.
 *
 * Ownership and execution
 *   - Every buffer is allocated by the caller.  Pointers named d_* or documented
 *     as "device" must be device memory of the current CUDA device; the library
 *     never allocates device memory, never synchronises the device, and enqueues
 *     work only on `stream` (a cudaStream_t passed as void*; NULL = legacy stream).
 *   - Device pointers must be 16-byte aligned; tensors are dense (no strides).
 *   - Functions are thread-safe; calls on one stream run in order.
 *
 * Errors
 *   Every int-returning function returns LLA_OK (0) or a negative code.  On error
 *   nothing was enqueued, and lla_last_error() (thread-local) describes it.
 *   Errors found on the device (positions outside the RoPE table, ctx_len outside
 *   [0, n_cap], cache slots outside the cache) never fault: the offending element
 *   is skipped or clamped and a bit is set in a device status word (see below).
 */
#ifndef LLA_H_
#define LLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LLA_OK 0
#define LLA_ERR_INVALID (-1)     /* null pointer, bad size, misaligned pointer, t >= T ... */
#define LLA_ERR_UNSUPPORTED (-2) /* shape outside the supported set (see lla_cfg) */
#define LLA_ERR_TOO_SMALL (-3)   /* packed / table / workspace buffer too small */
#define LLA_ERR_CUDA (-4)        /* a CUDA call or kernel launch failed */

#define LLA_MODE_PER_HEAD 0 /* one (c_k, c_v) pair per token, layer and head */
#define LLA_MODE_2D 1       /* LLA-2D: one (c_k, c_v) pair per token and layer */

/* Device status bits (see lla_decode_attn / lla_encode). */
#define LLA_STATUS_POSITION_RANGE 1 /* a history position or q_pos outside [0, rope_max_pos) */
#define LLA_STATUS_CTX_RANGE 2      /* ctx_len[b] outside [0, n_cap] (clamped) */
#define LLA_STATUS_SLOT_RANGE 4     /* an encode slot outside [0, n_slots) (skipped) */
#define LLA_STATUS_TIMEOUT 8        /* a kernel wait timed out; that call's output is invalid */

/*
 * Codec geometry of one shared layer.
 * Supported: 1 <= T <= 64; 1 <= H <= 128; d_head in {32, 64, 96, 128};
 * r_k, r_v multiples of 8 in [8, 256]; rope_base > 1; sm_scale >= 0;
 * d_rope in {0, 32, 64, d_head} (see the field).
 */
typedef struct lla_cfg {
  int32_t T;        /* loops */
  int32_t H;        /* attention heads (K/V heads; MHA) */
  int32_t d_head;   /* head width d */
  int32_t r_k;      /* K latent width */
  int32_t r_v;      /* V latent width */
  int32_t mode;     /* LLA_MODE_PER_HEAD or LLA_MODE_2D */
  float rope_base;  /* RoPE base, e.g. 10000 */
  float sm_scale;   /* softmax scale; 0 selects 1/sqrt(d_head) */
  int32_t d_rope;   /* 0: RoPE over the whole head (the method's default).  Otherwise the
                       decoupled RoPE of the close reading, Appendix J: only the first
                       d_rope dims of q and k rotate, as a rotary vector of their own width
                       (pairs (i, i + d_rope/2), angle pos * rope_base^(-2 i / d_rope)),
                       and the other dims form a NoPE content path that decode absorbs into
                       the query.  Supported: 32 or 64, below d_head, decode on the
                       tensor-core path (per head and LLA-2D); d_rope == d_head is the
                       default RoPE. */
} lla_cfg;

/* Last error message of the calling thread ("" if none). Never NULL. */
const char* lla_last_error(void);

/* Library version string ("lla-b200 <major>.<minor> ..."); 0.2 added lla_cfg.d_rope,
 * the full-memory fast path and the eviction calls. */
const char* lla_version(void);

/* ------------------------------------------------------------------------ */
/* Bookkeeping (host only, exact integers).                                  */
/* ------------------------------------------------------------------------ */

/*
 * Exact compression ratio of the persistent cache as a reduced fraction num/den.
 * Per head: 2 T d_head / (r_k + r_v)  (close reading §二.2 eq. (4); gist.science
 * "Zentrale Beiträge").  LLA-2D: 2 T H d_head / (r_k + r_v)  (close reading §二.6).
 */
int lla_ratio(const lla_cfg* cfg, int64_t* num, int64_t* den);

/*
 * Bytes of bf16 latent cache for `tokens` tokens over `layers` layers:
 * (r_k + r_v) * H * tokens * layers * 2 per head, (r_k + r_v) * tokens * layers * 2
 * for LLA-2D.  Also the uncompressed loop-indexed cache (2 T H d_head scalars per
 * token and layer) when teacher != 0.  Fails with LLA_ERR_INVALID on overflow.
 */
int lla_cache_bytes(const lla_cfg* cfg, int64_t tokens, int64_t layers, int teacher,
                    int64_t* bytes);

/* ------------------------------------------------------------------------ */
/* Codec packing (once per layer).                                            */
/* ------------------------------------------------------------------------ */

/* Size in bytes of the packed codec buffer for cfg (0 if cfg is unsupported). */
size_t lla_codec_packed_bytes(const lla_cfg* cfg);

/*
 * Pack fp32 codec parameters (device pointers) into the library's internal
 * device layout.  Inputs (row-major fp32):
 *   per head:  W_down_{k,v} [H][T*d][r],  W_up_{k,v} [H][T][d][r],  mu_{k,v} [H][T*d]
 *   LLA-2D:    W_down_{k,v} [T*H*d][r],   W_up_{k,v} [T][H][d][r],  mu_{k,v} [T*H*d]
 *   (concatenation order: loop-major, then head for LLA-2D, then the d entries.)
 * The packed buffer (`packed`, device, >= lla_codec_packed_bytes(cfg)) holds W_up
 * and mu in fp32, W_down rounded to bf16 (round to nearest even; stored twice: row
 * major, and cut into the tensor-core encode's operand tiles), and the encode bias
 * mu W_down computed with that rounded W_down.  Inputs may be freed once the stream
 * has passed this call.
 */
int lla_codec_pack(const lla_cfg* cfg, const float* W_down_k, const float* W_down_v,
                   const float* W_up_k, const float* W_up_v, const float* mu_k,
                   const float* mu_v, void* packed, size_t packed_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* RoPE table (once per d_head / base / maximum position).                    */
/* ------------------------------------------------------------------------ */

/* Size in bytes of the RoPE table covering positions [0, max_pos). */
size_t lla_rope_table_bytes(const lla_cfg* cfg, int32_t max_pos);

/*
 * Fill `table` (device) with (cos, sin) of pos * rope_base^(-2i/d_head) for
 * pos < max_pos, i < d_head/2, as fp32 pairs [max_pos][d_head/2][2].  Angles are
 * formed and reduced in fp64 and rounded once to fp32, so large positions keep
 * full fp32 accuracy (close reading §二.3: full-dimension RoPE on the rebuilt K).
 */
int lla_rope_table(const lla_cfg* cfg, int32_t max_pos, void* table, size_t table_bytes,
                   void* stream);

/* ------------------------------------------------------------------------ */
/* Encode: codec write of finished tokens.                                    */
/* ------------------------------------------------------------------------ */

/*
 * c = (x - mu) W_down, rounded to bf16, for n_tok finished tokens
 * (gist.science, Kernmechanismus, latent storage; close reading §二.6 for LLA-2D).
 *   x_k, x_v  device bf16 [n_tok][T][H][d]: each token's pre-RoPE K / V rows for all
 *             loops (the concatenation x = [x_0; ...; x_{T-1}] per head, or over
 *             (t, h) for LLA-2D).
 *   slot      device int64 [n_tok]: destination row of each token in the cache.
 *   c_k, c_v  device bf16 caches with n_slots rows: per head [n_slots][H][r_k] and
 *             [n_slots][H][r_v]; LLA-2D [n_slots][r_k] and [n_slots][r_v].  A
 *             cache laid out [B][n_cap][...] is addressed by slot = b * n_cap + j.
 *   status    optional device int32 (may be NULL): LLA_STATUS_SLOT_RANGE is OR-ed
 *             in when a slot is outside [0, n_slots); that token is skipped.
 * n_tok == 0 is a no-op.
 */
int lla_encode(const lla_cfg* cfg, const void* packed, int64_t n_tok, const uint16_t* x_k,
               const uint16_t* x_v, const int64_t* slot, int64_t n_slots, uint16_t* c_k,
               uint16_t* c_v, int32_t* status, void* stream);

/* ------------------------------------------------------------------------ */
/* Decode attention over the latent cache at loop t.                          */
/* ------------------------------------------------------------------------ */

/*
 * Workspace bytes needed by lla_decode_attn for (cfg, B, n_cap).  The workspace
 * must be zero-filled once before its first use; the library keeps it consistent
 * afterwards.  Its first two int32 words are the device status: word 0 collects
 * the bits of the call in flight, word 1 holds the final bits of the last
 * completed call (LLA_STATUS_* values).
 */
size_t lla_decode_workspace_bytes(const lla_cfg* cfg, int32_t B, int32_t n_cap);

/*
 * out[b][h] = attention of the loop-t query over the history rebuilt from the
 * latents plus the in-flight token (gist.science Kernmechanismus, loop-specific
 * reconstruction; close reading §二.3, RoPE after reconstruction):
 *   k_j  = RoPE(c_k,j W_up,k,t,h^T + mu_k,t,h, positions[b][j])
 *   s_j  = sm_scale * RoPE(q, q_pos[b]) . k_j ,  s_self likewise with k_self
 *   p    = softmax over {s_j : j < ctx_len[b]} and s_self
 *   out  = W_up,v,t,h (sum_j p_j c_v,j) + (sum_j p_j) mu_v,t,h + p_self v_self
 * (values are summed in latent space and up-projected once; equal to rebuilding
 * each V because the weights are linear in the rebuilt values.)
 *   packed        codec from lla_codec_pack (device)
 *   rope_table    table from lla_rope_table covering [0, rope_max_pos) (device)
 *   t             loop index, 0 <= t < T
 *   B, n_cap      batch and cache capacity per sequence (n_cap >= 0)
 *   ctx_len       device int32 [B]: history length of each sequence (<= n_cap)
 *   q, k_self, v_self  device fp32 [B][H][d]: the in-flight token's loop-t query,
 *                 key and value, pre-RoPE
 *   positions     device int32 [B][n_cap]: position of each history token
 *   q_pos         device int32 [B]: position of the in-flight token
 *   c_k, c_v      device bf16 latent caches: per head [B][n_cap][H][r_k] / [..][r_v];
 *                 LLA-2D [B][n_cap][r_k] / [B][n_cap][r_v].  Rows at or past ctx_len[b]
 *                 never reach the output, whatever they hold (NaN included).
 *   out           device fp32 [B][H][d]
 *   ws            device workspace of >= lla_decode_workspace_bytes(cfg, B, n_cap)
 * Work is launched on `stream` only; there is no host synchronisation.
 */
int lla_decode_attn(const lla_cfg* cfg, const void* packed, const void* rope_table,
                    int32_t rope_max_pos, int32_t t, int32_t B, int32_t n_cap,
                    const int32_t* ctx_len, const float* q, const float* k_self,
                    const float* v_self, const int32_t* positions, const int32_t* q_pos,
                    const uint16_t* c_k, const uint16_t* c_v, float* out, void* ws,
                    size_t ws_bytes, void* stream);

/*
 * lla_decode_attn for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this entry point; it exists for deployment.
 * Some callers cannot call cudaMalloc or any other allocator when they run
 * decode: code inside an allocator-free region of a host runtime, plugins that
 * are handed only their input and output buffers, or servers that forbid
 * allocation after start-up so that their memory use stays fixed.  This call
 * computes exactly what lla_decode_attn computes (same kernels, same arguments
 * and layouts) but takes no workspace: its split partials and status words live
 * in a fixed device array of 8 MiB (8388608 bytes) that the library holds on
 * every GPU where it is loaded, until the process exits.
 *   - Shapes whose workspace (lla_decode_workspace_bytes) exceeds 8 MiB are
 *     rejected with LLA_ERR_TOO_SMALL, and every argument lla_decode_attn checks
 *     is checked, before anything is enqueued: a rejected call leaves the array
 *     and status_out untouched.  B == 0 enqueues nothing.
 *   - The first call on a device looks up the array's device address with that
 *     device current (cudaGetSymbolAddress); make that first call before any
 *     stream capture.  Later calls reuse the address while the device keeps the
 *     same CUDA context, and look it up again after a device reset.
 *   - All calls share the one array and it keeps the last call's contents.  Each
 *     call clears the status words it needs; calls that overlap on the GPU (on
 *     different streams, or from different threads) race on the array and must
 *     be serialised by the caller.
 *   - status_out: optional device int32 (may be NULL) that receives this call's
 *     LLA_STATUS_* bits, written on `stream` after the kernels.
 * It allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
int lla_decode_attn_noalloc(const lla_cfg* cfg, const void* packed, const void* rope_table,
                            int32_t rope_max_pos, int32_t t, int32_t B, int32_t n_cap,
                            const int32_t* ctx_len, const float* q, const float* k_self,
                            const float* v_self, const int32_t* positions,
                            const int32_t* q_pos, const uint16_t* c_k, const uint16_t* c_v,
                            float* out, int32_t* status_out, void* stream);

/*
 * Number of kernel launches one lla_decode_attn call makes for (cfg, B, n_cap)
 * (for launch accounting by callers); -1 if the shape is unsupported.
 */
int lla_decode_launches(const lla_cfg* cfg, int32_t B, int32_t n_cap);

/* ------------------------------------------------------------------------ */
/*
 * Eviction composed with the latent cache: a sink + window retention budget
 * (close reading §四.10, Table 9: 4 sink tokens + a 256-token window; Appendix J:
 * a 1024-token budget).  The first `sink` history tokens and the `window` most
 * recent ones are kept, each at its own position.  A sequence's cache rows then
 * act as sink + window slots: history position p < sink lives in slot p, and
 * p >= sink in slot sink + (p - sink) mod window, overwriting the position that
 * just left the window.  Each slot's positions entry holds its token's position
 * and the decode reads slots [0, ctx_len) with ctx_len = min(n, sink + window);
 * attention over a set does not depend on slot order, so lla_decode_attn is
 * used unchanged.  No data moves when a token is evicted.
 */

/* Slot (row within its sequence) of history position pos; host only, exact.
 * Returns -1 when sink < 0, window < 1 or pos < 0. */
int64_t lla_evict_slot(int32_t sink, int32_t window, int64_t pos);

/*
 * Decode-time append under eviction, one new history token per sequence:
 *   pos        device int32 [B]: history position of each sequence's new token
 *              (its index in the history: the previous ctx_len when nothing was
 *              evicted yet); pos < 0 leaves the sequence untouched and writes
 *              slot -1 (lla_encode then skips it).
 *   slot       device int64 [B] (out): flat cache row b * n_cap + slot for lla_encode.
 *   positions  device int32 [B][n_cap] (in/out): the slot's entry is set to pos.
 *   ctx_len    device int32 [B] (out): min(pos + 1, sink + window).
 * Requires B >= 0, n_cap >= 1, sink >= 0, window >= 1 and sink + window <= n_cap
 * (LLA_ERR_INVALID otherwise); pointers 8-byte (slot) or 4-byte aligned.
 * Enqueued on `stream`; B == 0 is a no-op.
 */
int lla_evict_append(int32_t B, int32_t n_cap, int32_t sink, int32_t window, const int32_t* pos,
                     int64_t* slot, int32_t* positions, int32_t* ctx_len, void* stream);

/* ------------------------------------------------------------------------ */
/* Full-memory fast path: rebuild once, then ordinary attention.              */
/* ------------------------------------------------------------------------ */

/*
 * The close reading ("Looped Latent Attention: 跨循环 KV 压缩精读", §四.9, Table 5
 * and the paragraph after it) contrasts the latent store (keep only latents,
 * rebuild on every read) with a full-memory fast path that keeps the complete
 * rebuilt K/V, giving up the cache saving for speed.  Per §二.3 the codec works
 * on pre-RoPE K and the model rotates the rebuilt key at its position before it
 * is cached, so the full cache holds rotated keys.
 *
 * Full cache of one loop t: k_full and v_full, each device bf16 [B][H][n_cap][d]
 * (head-major: one (sequence, head) history is a contiguous run of rows).
 */

/* Bytes of one of k_full / v_full for (cfg, B, n_cap); 0 if the arguments are invalid. */
size_t lla_full_kv_bytes(const lla_cfg* cfg, int32_t B, int32_t n_cap);

/*
 * Rebuild rows of the loop-t full cache from the latent cache:
 *   k_full[b][h][j] = bf16(RoPE(c_k[b][j](h) W_up,k,t,h^T + mu_k,t,h, positions[b][j]))
 *   v_full[b][h][j] = bf16(c_v[b][j](h) W_up,v,t,h^T + mu_v,t,h)
 * for each row b * n_cap + j listed in slot[0 .. n_rows) (device int64), or for
 * rows 0 .. n_rows-1 when slot is NULL (n_rows <= B * n_cap; B * n_cap rebuilds the
 * whole cache once).  c_k, c_v and positions are laid out as for lla_decode_attn;
 * packed and rope_table as for lla_decode_attn.  status (optional device int32)
 * collects LLA_STATUS_SLOT_RANGE (a slot outside [0, B * n_cap): skipped) and
 * LLA_STATUS_POSITION_RANGE (a position outside the table: clamped).  Runs on the
 * CUDA cores; it is a once-per-token conversion, not a per-step cost.
 */
int lla_full_rebuild(const lla_cfg* cfg, const void* packed, const void* rope_table,
                     int32_t rope_max_pos, int32_t t, int32_t B, int32_t n_cap,
                     const int32_t* positions, const uint16_t* c_k, const uint16_t* c_v,
                     const int64_t* slot, int64_t n_rows, uint16_t* k_full, uint16_t* v_full,
                     int32_t* status, void* stream);

/* Workspace bytes for lla_full_decode_attn (zero-filled once before first use; its
 * first two int32 words are the status words described at lla_decode_workspace_bytes). */
size_t lla_full_decode_workspace_bytes(const lla_cfg* cfg, int32_t B, int32_t n_cap);

/* Kernel launches one lla_full_decode_attn call makes (1 or 2), or -1 if invalid. */
int lla_full_decode_launches(const lla_cfg* cfg, int32_t B, int32_t n_cap);

/*
 * out[b][h] = ordinary decode attention over the full cache plus the in-flight token:
 *   s_j   = sm_scale * RoPE(q, q_pos[b]) . k_full[b][h][j]   (j < ctx_len[b])
 *   s_self = sm_scale * RoPE(q, q_pos[b]) . RoPE(k_self, q_pos[b])
 *   out   = sum_j p_j v_full[b][h][j] + p_self v_self,  p = softmax(s, s_self)
 *   q, k_self, v_self  device fp32 [B][H][d], pre-RoPE; q_pos, ctx_len device int32 [B]
 *   k_full, v_full     device bf16 [B][H][n_cap][d] (may be NULL when n_cap == 0)
 *   out                device fp32 [B][H][d]
 * The cfg's codec fields (T, r_k, r_v, mode) are not used.  B * H * n_cap must stay
 * below 2^31 rows (LLA_ERR_UNSUPPORTED otherwise).  Device-side range problems set
 * LLA_STATUS_POSITION_RANGE / LLA_STATUS_CTX_RANGE in the workspace status word.
 */
int lla_full_decode_attn(const lla_cfg* cfg, const void* rope_table, int32_t rope_max_pos,
                         int32_t B, int32_t n_cap, const int32_t* ctx_len, const float* q,
                         const float* k_self, const float* v_self, const int32_t* q_pos,
                         const uint16_t* k_full, const uint16_t* v_full, float* out, void* ws,
                         size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LLA_H_ */
