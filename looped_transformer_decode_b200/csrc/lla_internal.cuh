// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "lla.h"

namespace lla {

// Status words at the head of the decode workspace: [0] bits of the call in
// flight, [1] bits of the last completed call.  Partials start at kWsHeader.
constexpr size_t kWsHeader = 256;
constexpr int kTile = 128;          // history tokens per tile (one per thread / TMEM lane)
constexpr int kMaxSplits = 64;      // context splits per (b, h) at most

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// SMs of the current device, which sizes every persistent grid and split plan.
// Without a usable device (host-only use of the sizing calls) a B200's 148.
int sm_count();

// Offsets (bytes) of each section of the packed codec buffer.
//   wup_k      fp32 [T][H][d][r]      loop-t, head-h up-projection W_up,k,t,h (d x r)
//   wup_v      fp32 [T][H][r][d]      W_up,v,t,h transposed (read column-wise by the combine)
//   mu_{k,v}   fp32 [T][H][d]         loop-t, head-h mean slice mu_t,h
//   wd_{k,v}   bf16 [L][r][W]         W_down^T (rows = latent index), L = H (per head) or 1
//   bias_{k,v} fp32 [L][r]            mu W_down with the bf16-rounded W_down
//   wimg_{k,v} bf16 [L][W/kc][N][kc]  the same W_down^T cut into K chunks of kc entries,
//                                     each chunk the swizzled K-major operand image of
//                                     the tensor-core encode (N = r rounded up to 16,
//                                     rows >= r zero), so that one bulk copy stages it
struct PackedLayout {
  size_t wupk, wupv, muk, muv, wdk, wdv, biask, biasv, wimgk, wimgv, total;
  int L;     // latents per token and layer: H (per head) or 1 (LLA-2D)
  int W;     // encode input width: T*d (per head) or T*H*d (LLA-2D)
};

PackedLayout packed_layout(const lla_cfg& c);

// K chunk (entries) of the tensor-core encode: 64 (128-byte swizzle) when a head's
// d entries (per head) or the whole input row (LLA-2D) split into 64s, else 32
// (64-byte swizzle).  Every supported d is a multiple of 32.
inline int encode_kc(const lla_cfg& c) {
  const int unit = c.mode == LLA_MODE_PER_HEAD ? c.d_head : c.T * c.H * c.d_head;
  return unit % 64 == 0 ? 64 : 32;
}
inline int pad16(int r) { return (r + 15) / 16 * 16; }
// Dims of q and k that RoPE rotates: the whole head, or the decoupled branch.
inline int rotary_dims(const lla_cfg& c) { return c.d_rope ? c.d_rope : c.d_head; }
// Decoupled RoPE with a NoPE content path (d_rope below d_head).
inline bool has_nope(const lla_cfg& c) { return c.d_rope != 0 && c.d_rope < c.d_head; }

// Decode split plan shared by the workspace sizing and the launcher.
struct SplitPlan {
  int n_tiles;          // ceil(n_cap / kTile)
  int splits;           // S
  int tiles_per_split;  // tiles handled by one CTA
  bool tensor_cores;    // the tcgen05 partial kernel takes this shape
  size_t ops_bytes;     // workspace for its per-(b, h) operand images
};
SplitPlan split_plan(const lla_cfg& c, int B, int n_cap);
size_t partials_bytes(const lla_cfg& c, int B, int S);

// Every host check lla_decode_attn makes before it enqueues work, except those of
// the workspace.  Returns LLA_OK (also for B == 0, which enqueues nothing), or the
// error code with lla_last_error() set.
int decode_check_args(const lla_cfg* cfg, const void* packed, const void* rope_table,
                      int32_t rope_max_pos, int32_t t, int32_t B, int32_t n_cap,
                      const int32_t* ctx_len, const float* q, const float* k_self,
                      const float* v_self, const int32_t* positions, const int32_t* q_pos,
                      const uint16_t* c_k, const uint16_t* c_v, const float* out);

// Kernel launchers (return cudaError_t of the launch).
cudaError_t launch_rope_table(const lla_cfg& c, int max_pos, float2* table, cudaStream_t s);
cudaError_t launch_pack(const lla_cfg& c, const PackedLayout& L, const float* wdk,
                        const float* wdv, const float* wupk, const float* wupv,
                        const float* muk, const float* muv, char* packed, cudaStream_t s);
cudaError_t launch_encode(const lla_cfg& c, const PackedLayout& L, const char* packed,
                          int64_t n_tok, const __nv_bfloat16* xk, const __nv_bfloat16* xv,
                          const int64_t* slot, int64_t n_slots, __nv_bfloat16* ck,
                          __nv_bfloat16* cv, int32_t* status, cudaStream_t s);
// Same contract on the tensor cores; cudaErrorNotSupported leaves the call to launch_encode.
cudaError_t launch_encode_tc(const lla_cfg& c, const PackedLayout& L, const char* packed,
                             int64_t n_tok, const __nv_bfloat16* xk, const __nv_bfloat16* xv,
                             const int64_t* slot, int64_t n_slots, __nv_bfloat16* ck,
                             __nv_bfloat16* cv, int32_t* status, cudaStream_t s);

// Eviction (sink + window slots over the latent cache).
int64_t evict_slot(int32_t sink, int32_t window, int64_t pos);
cudaError_t launch_evict_append(int B, int n_cap, int sink, int window, const int32_t* pos,
                                int64_t* slot, int32_t* positions, int32_t* ctx_len,
                                cudaStream_t s);

struct DecodeArgs {
  int T, H, d, r_k, r_v, mode;
  int rd;                // rotated dims: d, or the decoupled rotary branch's d_rope
  float kappa;           // sm_scale * log2(e): scores are kept in base-2 units
  int t, B, n_cap, rope_max_pos;
  float rope_base;
  const float* wupk_t;   // packed W_up,k at loop t: [H][d][r_k]
  const float* wupv_t;   // [H][r_v][d] (transposed)
  const float* muk_t;    // [H][d]
  const float* muv_t;    // [H][d]
  const float2* rope;    // [rope_max_pos][d/2]
  const int32_t* ctx_len;
  const float* q;
  const float* k_self;
  const float* v_self;
  const int32_t* positions;
  const int32_t* q_pos;
  const __nv_bfloat16* ck;
  const __nv_bfloat16* cv;
  long long lat_tok_k, lat_tok_v;    // elements between consecutive tokens of one sequence
  long long lat_head_k, lat_head_v;  // elements between heads (0 for LLA-2D)
  float* out;
  int32_t* status;       // ws words [0], [1]
  float* partials;       // [B][H][S][2 + r_v]
  int S, tiles_per_split;
  unsigned char* ops;    // per-(b, h) MMA operand images (tensor-core path), or null
  uint32_t* counters;    // [B * H + 1]; word B * H counts finished CTAs (fused combine), or null
};
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s, int* launches);
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s);

// Tensor-core (tcgen05) partial kernel for per-head decode.  decode_tc_plan
// reports whether the shape takes that path and its context split; the launcher
// returns cudaErrorNotSupported when it cannot run the shape.
bool decode_tc_plan(const lla_cfg& c, int B, int n_cap, int* S, int* tps, size_t* ops_bytes);
cudaError_t launch_decode_tc(const lla_cfg& c, const DecodeArgs& a, cudaStream_t s);

// Full-memory fast path: the loop-t K/V rebuilt once into a full bf16 cache
// [B][H][n_cap][d] (keys rotated), and ordinary decode attention over it.
struct FullRebuildArgs {
  int d, H, r_k, r_v, B, n_cap, rope_max_pos;
  long long n_rows;
  const int64_t* slot;             // [n_rows] rows b * n_cap + j, or null: rows 0 .. n_rows-1
  const int32_t* positions;        // [B][n_cap]
  const float2* rope;              // [rope_max_pos][d/2]
  const float* wupk_t;             // [H][d][r_k] at loop t
  const float* wupv_t;             // [H][r_v][d]
  const float* muk_t;              // [H][d]
  const float* muv_t;
  const __nv_bfloat16* ck;
  const __nv_bfloat16* cv;
  long long lat_tok_k, lat_tok_v, lat_head_k, lat_head_v;
  __nv_bfloat16* k_full;
  __nv_bfloat16* v_full;
  int32_t* status;                 // optional
};
struct FullDecodeParams {
  int B, H, n_cap, d, S, tps, n_items, rope_max_pos, fuse;
  float kappa;
  const float* q;
  const float* k_self;
  const float* v_self;
  const int32_t* q_pos;
  const int32_t* ctx_len;
  const float2* rope;
  float* out;
  float* partials;                 // [B][H][S][2 + d] when S > 1
  int32_t* status;                 // ws words [0], [1]
  uint32_t* counter;               // ws word [4]: CTAs finished in this call
};
struct FullPlan {
  int S = 1, tps = 1, grid = 1, grid_max = 148;
  long long n_items = 0;
};
FullPlan full_plan(const lla_cfg& c, int B, int n_cap);
cudaError_t launch_full_rebuild(const FullRebuildArgs& a, cudaStream_t s);
cudaError_t launch_full_decode(const FullDecodeParams& p, const void* k_full, const void* v_full,
                               int grid, cudaStream_t s);

// Record `fmt` as the calling thread's lla_last_error() message; returns `code`.
int set_error(int code, const char* fmt, ...);

}  // namespace lla
