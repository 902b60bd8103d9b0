// LLA decode attention on the 5th-generation tensor cores (sm_100a), per head and
// LLA-2D.  In LLA-2D every head reads the same latent row (close reading §二.6),
// so a work item's heads share each latent tile.
//
// Same arithmetic as the CUDA-core kernel (query folded into the K
// up-projection, RoPE as a complex product, base-2 online softmax, V summed in
// latent space), organised for B200:
//
//   * decode_prep_kernel builds, per (b, h), the query-absorbed score operand
//     A~ = kappa conj(q~) W~ (and the bias M~, bf16 hi + lo) as the byte image of
//     the MMA's shared-memory operand; with decoupled RoPE it also writes the
//     NoPE content row;
//   * persistent CTAs, one per SM, walk a list of work items (sequence b, group
//     of heads, context split s); a TMA producer warp streams 128-token c_k tiles
//     into a swizzled K-major ring (and each item's operand images with one bulk
//     copy), another the c_v tiles into an MN-major ring;
//   * one warp issues the score tcgen05.mma U = C_k A~^T (+ the bias through a
//     ones column) into fp32 TMEM; the epilogue warpgroups read U, turn the RoPE
//     pairs at each token's position (complex factors advanced tile to tile),
//     run the online softmax and write the weights as bf16 hi + lo rows;
//   * another warp issues the V MMAs that accumulate sum_j p_j c_v,j in TMEM
//     (per head: P x C_v; LLA-2D: transposed, C_v^T P^T for all heads at once);
//   * with one split per head group the item is finished in the kernel (merge
//     with the in-flight token, W_up,v up-projection); otherwise split partials
//     go to decode_combine_kernel.
// The close reading §二.3 fixes the order (rebuild K, then RoPE at its
// position); folding q into W_up and RoPE into a complex dot product changes
// only the order of the same sums.
//
// Every wait is bounded (lla_sm100.cuh); on a timeout the CTA records
// LLA_STATUS_TIMEOUT, drains its in-flight copies, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "lla_internal.cuh"
#include "lla_sm100.cuh"

namespace lla {

namespace {

using namespace sm100;

constexpr int kEpiWG = 2;                       // epilogue warpgroups
constexpr int kEpiThreads = 128 * kEpiWG;       // warps 2 .. 2 + 4 kEpiWG - 1
constexpr int kEpiWarps = kEpiThreads / 32;
// warp 0: c_k producer, warp 1: score MMA issuer, warps 2..9: epilogue,
// warp 10: c_v producer, warp 11: V MMA issuer
constexpr int kThreads = 64 + kEpiThreads + 64;
constexpr int kVProdWarp = 2 + kEpiWarps, kVMmaWarp = 3 + kEpiWarps;
constexpr uint32_t kSmemLimit = 232448;  // per-block dynamic shared memory on sm_100

struct TcParams {
  int H, r_k, r_v, K_pad, box_k, nkb, swz;   // K latent tiles: K-major, swizzle code swz
  int lat_hk, lat_hv;                        // latent columns between heads (0: LLA-2D, shared)
  int nst_v;                                 // V latent ring depth (nst: K latent ring)
  uint32_t stv_off, stv_bytes, tx_v;
  int N_v, cvb, nvb, swz_v;                  // V latent tiles: MN-major boxes of cvb dims
  int nmb;                                   // 128-dim blocks of the V latent (V MMA rows)
  int B, n_cap, S, tps, HG, n_items, rope_max_pos;
  uint32_t st_off, st_bytes, cv_off, box_bytes, vbox_bytes;
  uint32_t b_off, b_head_bytes, b_sbo, bias_head_bytes, ones_off, bias_off, sbuf_off, p_off,
      red_off, ctx_off, rope_off, bar_off, misc_off;
  int nst, nacc, acc_cols, v_col0, tmem_cols;
  uint32_t tx_bytes;
  // LLA-2D kernel: B-operand buffers, P rows (N of the V MMA), 128-row blocks of r_v
  int nbuf_b, n_p, m_v;
  int poll;                                  // per-head hand-offs poll instead of suspending
  uint32_t nap_ns, enap_ns;                  // naps between polls: MMA issuers, epilogue
  uint32_t cnap_ns;                          // MMA issuers of a CTA whose phase tiles are all computed
  uint32_t spins;                            // polls before the first nap
  // fused split combine (per-head kernel): the CTA that finishes a group's last split
  // merges the splits, adds the in-flight token and up-projects with W_up,v
  const float* q;                            // [B][H][d]
  const float* k_self;
  const float* v_self;
  const float* wupv_t;                       // [H][r_v][d] at loop t
  const float* muv_t;                        // [H][d]
  float* out;                                // [B][H][d]
  float kappa;
  int d;
  uint32_t* counters;                        // word B * H: CTAs done (fused combine); rest unused
  uint32_t comb_off;                         // smem: olat [r_v], split weights [64], reductions
  int fuse_combine;                          // 1: the combine is done here (one split per group)
  uint32_t p_buf_bytes;
  // phase-operand kernel (decode_tcf_kernel): ne buffers of the phase operand E
  // ([128 tokens x d] bf16 each), F columns n_f = G r_k + 16, bytes of one item's
  // operand image, and the swizzle mask of the K latent tile (7: 128-byte rows,
  // 3: 64-byte rows)
  uint32_t e_off, e_bytes, b_img_bytes;
  int ne, n_f, kswz_mask;
  // phase table (phase-operand kernel): tile_p0[b][tile] is the position of the tile's
  // first token when its tokens sit at consecutive positions inside the table, whose
  // row p holds conj(e^{i p theta_i}) as bf16 pairs; -1 (or no table) otherwise
  const int32_t* tile_p0;
  int n_tiles_cap;                           // tiles per sequence: ceil(n_cap / 128)
  const float2* rope;    // [rope_max_pos][d/2]
  const int32_t* ctx_len;
  const int32_t* positions;
  const unsigned char* ops_b;     // [B][H] images of the MMA B operand
  const unsigned char* ops_bias;  // [B][H] images of the bias tile
  int32_t* status;
  float* partials;       // [B][H][S][2 + r_v]
  // theta_i / (2 pi) as 64-bit fixed-point fractions of a turn, per RoPE pair i
  uint32_t phi_lo[64], phi_hi[64];
  // conj(e^{i 128 theta_i}): advances conj(e^{i p theta_i}) by one tile of positions
  float2 step[64];
};

// compile-time value passed to generic lambdas
template <int V>
struct IntTag {
  static constexpr int value = V;
};
// how the phase-operand kernel's epilogue gets its phase tiles
constexpr int kPhaseComputed = 0, kPhaseMixed = 1, kPhaseTable = 2;

constexpr int kNoPos = -2147483647 - 1;       // raw position of a row past the context
constexpr int kReseedTiles = 32;              // exact RoPE factors at least this often

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  memcpy(&ra, &a, 8);
  memcpy(&rb, &b, 8);
  memcpy(&rc, &c, 8);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  float2 d;
  memcpy(&d, &rd, 8);
  return d;
}

// (cos, -sin) of pos * theta_i, i.e. conj(e^{i pos theta_i}).  The angle is reduced exactly in integer arithmetic
// (pos * phi_i mod 1 turn, phi_i = theta_i / 2pi in 0.64 fixed point), so the
// fp32 sine and cosine see an argument in [-pi, pi) with error below 1e-7 rad at
// any position.
__device__ __forceinline__ float2 rope_factor(uint32_t pos, uint32_t phi_lo, uint32_t phi_hi) {
  const uint32_t turns = pos * phi_hi + __umulhi(pos, phi_lo);
  const float ang = static_cast<float>(static_cast<int32_t>(turns)) * 1.46291807926715968e-9f;
  float sn, cs;
  __sincosf(ang, &sn, &cs);
  return make_float2(cs, -sn);
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// bar.red.or over the 128 threads of one warpgroup (named barrier `id`).
__device__ __forceinline__ int wg_barrier_or(uint32_t id, int pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.red.or.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(out)
      : "r"(pred), "r"(id)
      : "memory");
  return static_cast<int>(out);
}

// bar.red.or over NT epilogue threads (named barrier 1): returns the OR of `pred`.
template <int NT>
__device__ __forceinline__ int epi_barrier_or_n(int pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.red.or.pred po, 1, %2, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(out)
      : "r"(pred), "n"(NT)
      : "memory");
  return static_cast<int>(out);
}

// bar.red.or over the epilogue threads (named barrier 1): returns the OR of `pred`.
__device__ __forceinline__ int epi_barrier_or(int pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "barrier.red.or.pred po, 1, %2, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(out)
      : "r"(pred), "n"(kEpiThreads)
      : "memory");
  return static_cast<int>(out);
}

// registers -> TMEM, 16 consecutive columns (32x32b shape).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

__device__ __forceinline__ void tmem_ld2(uint32_t taddr, float* v) {
  uint32_t r0, r1;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(taddr));
  v[0] = __uint_as_float(r0);
  v[1] = __uint_as_float(r1);
}

__device__ __forceinline__ void tmem_st2(uint32_t taddr, float v0, float v1) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1,%2};" ::"r"(taddr),
               "r"(__float_as_uint(v0)), "r"(__float_as_uint(v1))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// TMEM -> registers, 8 consecutive columns (32x32b shape).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Slot of a ring of n entries and the parity of its current pass, stepped by one
// (no division per step).
struct RingPos {
  uint32_t slot = 0, phase = 0;
  __device__ __forceinline__ void next(uint32_t n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

struct ItemRange {
  int b, hg, s, tok0, tok_end, ntiles;
};

constexpr int kCtxCache = 1024;   // sequences whose context length is cached in smem

// ctx_s: clamped context lengths cached in shared memory (B <= kCtxCache), else null.
__device__ __forceinline__ ItemRange item_range(const TcParams& p, const int* ctx_s, int item,
                                                bool flag_ctx) {
  ItemRange r;
  r.s = item % p.S;
  const int u = item / p.S;
  r.hg = u % p.HG;
  r.b = u / p.HG;
  int n;
  if (ctx_s) {
    n = ctx_s[r.b];
  } else {
    n = p.ctx_len[r.b];
    if (n < 0 || n > p.n_cap) {
      if (flag_ctx) atomicOr(p.status, LLA_STATUS_CTX_RANGE);
      n = n < 0 ? 0 : p.n_cap;
    }
  }
  r.tok0 = r.s * p.tps * kTile;
  r.tok_end = min(r.tok0 + p.tps * kTile, n);
  r.ntiles = r.tok_end > r.tok0 ? (r.tok_end - r.tok0 + kTile - 1) / kTile : 0;
  return r;
}

// Walks this CTA's tiles in processing order (items with no tiles are skipped).
struct TileCursor {
  int item, k;
  ItemRange r;
  bool valid;
};

__device__ __forceinline__ void cursor_first(const TcParams& p, const int* ctx_s, TileCursor& c) {
  c.valid = false;
  c.k = 0;
  for (c.item = blockIdx.x; c.item < p.n_items; c.item += gridDim.x) {
    c.r = item_range(p, ctx_s, c.item, false);
    if (c.r.ntiles > 0) {
      c.valid = true;
      return;
    }
  }
}

__device__ __forceinline__ void cursor_next(const TcParams& p, const int* ctx_s, TileCursor& c) {
  if (!c.valid) return;
  if (++c.k < c.r.ntiles) return;
  c.k = 0;
  for (c.item += gridDim.x; c.item < p.n_items; c.item += gridDim.x) {
    c.r = item_range(p, ctx_s, c.item, false);
    if (c.r.ntiles > 0) return;
  }
  c.valid = false;
}

// Raw position of token `row` of the cursor's tile (0 for rows past the context).
// The range check is left to the consumer so that the load does not stall here.
__device__ __forceinline__ int cursor_pos(const TcParams& p, const TileCursor& c, int row) {
  if (!c.valid) return kNoPos;
  const int t0 = c.r.tok0 + c.k * kTile;
  if (row >= c.r.tok_end - t0) return kNoPos;
  return p.positions[(size_t)c.r.b * p.n_cap + t0 + row];
}

// Table mark of the cursor's tile: the position of its first token when the prep grid
// found the tile's positions consecutive inside the phase table, else -1 (and -1
// without a table or past the last tile).
__device__ __forceinline__ int cursor_tp0(const TcParams& p, const TileCursor& c) {
  if (!p.tile_p0 || !c.valid) return -1;
  return __ldcg(p.tile_p0 + (size_t)c.r.b * p.n_tiles_cap + c.r.s * p.tps + c.k);
}

__device__ __forceinline__ int checked_pos(const TcParams& p, int pos) {
  if (pos < 0 || pos >= p.rope_max_pos) {
    atomicOr(p.status, LLA_STATUS_POSITION_RANGE);
    return 0;
  }
  return pos;
}

// Builds, for every (b, h), the MMA B operand A~ (rows n = 2i: Re, 2i+1: Im of the
// query-absorbed up-projection, K = latent index) as the byte image of the
// no-swizzle K-major shared-memory layout, and the bias tile image (K column 0 =
// bf16 hi part of M~, column 1 = lo part).  One CTA of 128 threads per (h, b).
template <int D>
// D: rotated dims (the head, or the decoupled rotary branch).  With decoupled RoPE
// (d_full > D) the images get 16 more rows: row D is the NoPE content path with the
// query absorbed, kappa sum_{e >= D} q_e W_up,k[e][k] (bias kappa q_nope . mu_nope),
// and rows D + 1 .. D + 15 are zero.
__global__ void __launch_bounds__(128) decode_prep_kernel(
    const float* __restrict__ q, const int32_t* __restrict__ q_pos, const float2* __restrict__ rope,
    int rope_max_pos, const float* __restrict__ wupk_t, const float* __restrict__ muk_t, float kappa,
    int H, int r_k, int K_pad, unsigned char* __restrict__ ops_b,
    unsigned char* __restrict__ ops_bias, int32_t* status, uint32_t* counters, int d_full) {
  constexpr int HALF = D / 2;
  const int NS = d_full > D ? D + 16 : D;      // rows of the images
  // the partial kernel may start its prologue and latent loads now; it waits for
  // this grid before it reads the images or the counter
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float2 qc[HALF];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  // the CTA counter of the fused-combine kernels starts every call at zero (this
  // kernel runs first)
  if (counters && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && tid == 0)
    counters[(size_t)gridDim.y * H] = 0u;
  // This thread's first image chunk and first bias chunk need nothing from the query:
  // their W_up,k and mu values are read before the query's RoPE factors (which wait
  // for q_pos), so the two reads overlap.
  const float* W = wupk_t + (size_t)h * d_full * r_k;  // [d][r_k]
  const float* mu = muk_t + (size_t)h * d_full;
  const int chunks = D * K_pad / 8;
  const int c_first = blockIdx.z * blockDim.x + tid;
  float w_first[16];
  if (c_first < chunks) {
    const int n = (c_first / K_pad) * 8 + (c_first & 7), k0 = ((c_first >> 3) % (K_pad / 8)) * 8;
    const int i = n >> 1;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const bool in = k0 + e < r_k;
      w_first[2 * e] = in ? W[(size_t)i * r_k + k0 + e] : 0.f;
      w_first[2 * e + 1] = in ? W[(size_t)(i + HALF) * r_k + k0 + e] : 0.f;
    }
  }
  float mu_first[2] = {0.f, 0.f};
  if (c_first < D * 2 && ((c_first >> 3) & 1) == 0) {
    const int i = ((c_first >> 4) * 8 + (c_first & 7)) >> 1;
    mu_first[0] = mu[i];
    mu_first[1] = mu[i + HALF];
  }
  int qp = q_pos[b];
  if (qp < 0 || qp >= rope_max_pos) {
    if (tid == 0 && h == 0 && blockIdx.z == 0) atomicOr(status, LLA_STATUS_POSITION_RANGE);
    qp = 0;
  }
  const float* qh = q + ((size_t)b * H + h) * d_full;
  for (int i = tid; i < HALF; i += blockDim.x) {
    const float2 e = rope[(size_t)qp * HALF + i];
    const float x0 = qh[i], x1 = qh[i + HALF];
    qc[i] = make_float2(x0 * e.x - x1 * e.y, x0 * e.y + x1 * e.x);
  }
  __syncthreads();
  unsigned char* img = ops_b + ((size_t)b * H + h) * (size_t)NS * K_pad * 2;
  // One 16-byte chunk (8 consecutive K values of one row n) per iteration; rows < D
  // here, the 16 NoPE rows (decoupled RoPE) below.
  for (int c = c_first; c < chunks; c += gridDim.z * blockDim.x) {
    const int n = (c / K_pad) * 8 + (c & 7);
    const int k0 = ((c >> 3) % (K_pad / 8)) * 8;
    __align__(16) __nv_bfloat16 v[8];
    const int i = n >> 1;
    const float2 z = qc[i];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int k = k0 + e;
      float val = 0.f;
      if (k < r_k) {
        const float wr = c == c_first ? w_first[2 * e] : W[(size_t)i * r_k + k];
        const float wi = c == c_first ? w_first[2 * e + 1] : W[(size_t)(i + HALF) * r_k + k];
        val = (n & 1) ? kappa * (z.x * wi - z.y * wr) : kappa * (z.x * wr + z.y * wi);
      }
      v[e] = __float2bfloat16_rn(val);
    }
    *reinterpret_cast<uint4*>(img + (size_t)c * 16) = *reinterpret_cast<const uint4*>(v);
  }
  __shared__ float a_part[4][256];
  __shared__ float q_nope[128];
  __shared__ float mu_nope;
  if (d_full > D && blockIdx.z == 0) {
    // NoPE content path: the query absorbed into the unrotated dims' up-projection,
    // a[k] = kappa sum_{dd >= D} q_dd W[dd][k], and its bias kappa q_nope . mu_nope.
    // Warp w sums a quarter of the dims for every k (lanes over k: coalesced W rows).
    const int nd = d_full - D, w = tid >> 5, lane = tid & 31;
    for (int dd = tid; dd < nd; dd += blockDim.x) q_nope[dd] = qh[D + dd];
    __syncthreads();
    const int per = (nd + 3) / 4, d0 = w * per, d1 = min(nd, d0 + per);
    for (int k = lane; k < r_k; k += 32) {
      float acc = 0.f;
#pragma unroll 8
      for (int dd = d0; dd < d1; ++dd) acc = fmaf(q_nope[dd], W[(size_t)(D + dd) * r_k + k], acc);
      a_part[w][k] = acc;
    }
    if (tid < 32) {
      float acc = 0.f;
      for (int dd = tid; dd < nd; dd += 32) acc = fmaf(q_nope[dd], muk_t[(size_t)h * d_full + D + dd], acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (tid == 0) mu_nope = kappa * acc;
    }
    __syncthreads();
    // rows D .. D + 15: two 8-row groups of K_pad / 8 chunks each; only row D is nonzero
    for (int c2 = tid; c2 < 2 * K_pad; c2 += blockDim.x) {
      const int c = (D / 8) * K_pad + c2;
      const int n = (c / K_pad) * 8 + (c & 7);
      const int k0 = ((c >> 3) % (K_pad / 8)) * 8;
      __align__(16) __nv_bfloat16 v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        v[e] = __float2bfloat16_rn(n == D && k0 + e < r_k
                                       ? kappa * ((a_part[0][k0 + e] + a_part[1][k0 + e]) +
                                                  (a_part[2][k0 + e] + a_part[3][k0 + e]))
                                       : 0.f);
      *reinterpret_cast<uint4*>(img + (size_t)c * 16) = *reinterpret_cast<const uint4*>(v);
    }
  }
  // Bias tile image [D x 16]: chunk c covers row n = (c / 2 / 8) * 8 + c % 8 ... laid out as
  // core matrices (n / 8, k / 8) at (n / 8) * 256 + (k / 8) * 128 + (n % 8) * 16.
  unsigned char* bimg = ops_bias + ((size_t)b * H + h) * (size_t)NS * 32;
  for (int c = c_first; c < D * 2; c += gridDim.z * blockDim.x) {
    const int n = (c >> 4) * 8 + (c & 7);
    const int kc = (c >> 3) & 1;
    __align__(16) __nv_bfloat16 v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __float2bfloat16_rn(0.f);
    if (kc == 0) {
      const int i = n >> 1;
      const float2 z = qc[i];
      const float mr = c == c_first ? mu_first[0] : mu[i];
      const float mi = c == c_first ? mu_first[1] : mu[i + HALF];
      const float val = (n & 1) ? kappa * (z.x * mi - z.y * mr) : kappa * (z.x * mr + z.y * mi);
      v[0] = __float2bfloat16_rn(val);
      v[1] = __float2bfloat16_rn(val - __bfloat162float(v[0]));
    }
    *reinterpret_cast<uint4*>(bimg + (size_t)c * 16) = *reinterpret_cast<const uint4*>(v);
  }
  if (d_full > D && blockIdx.z == 0) {
    // bias rows D .. D + 15: row D carries kappa q_nope . mu_nope as bf16 hi + lo
    for (int c = 2 * D + tid; c < 2 * NS; c += blockDim.x) {
      const int n = (c >> 4) * 8 + (c & 7);
      __align__(16) __nv_bfloat16 v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __float2bfloat16_rn(0.f);
      if (n == D && ((c >> 3) & 1) == 0) {
        v[0] = __float2bfloat16_rn(mu_nope);
        v[1] = __float2bfloat16_rn(mu_nope - __bfloat162float(v[0]));
      }
      *reinterpret_cast<uint4*>(bimg + (size_t)c * 16) = *reinterpret_cast<const uint4*>(v);
    }
  }
}

// Before the CTA frees TMEM: arrive on `bar` once every MMA this thread issued has
// completed, and wait for that (bounded).  In a normal run they all have completed
// already (the epilogue waited on their commits); after an abort some may not have.
__device__ __forceinline__ void mma_drain(uint64_t* bar) {
  mma_commit(bar);
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, 0) && global_timer_ns() - t0 < kWaitTimeoutNs) {
  }
}

// log2 of the largest softmax weight a tile may carry before the V accumulator
// is rescaled to a new reference maximum.
constexpr float kRescaleLog2 = 8.f;

// Split combine of head (b, h), run by the 128 threads of one warpgroup (named
// barrier `bar`): merge the S split partials (m, l, sum p c_v) at a common
// maximum, add the in-flight token (its score q . k_self needs no rotation: both
// sit at q_pos), and o = W_up,v (sum p c_v) / l + (sum_hist p / l) mu_v + (p_self / l)
// v_self.  Same arithmetic as decode_combine_kernel.  Partials written by other
// CTAs are read past L1 (ld.global.cg).
__device__ void combine_head(const TcParams& p, int b, int h, unsigned char* scratch, int tid,
                             uint32_t bar) {
  float* olat = reinterpret_cast<float*>(scratch);   // [r_v]
  float* wts = olat + 256;                            // [64] split weights
  float* red = wts + 64;                              // [8]
  const int lane = tid & 31, w = tid >> 5;
  const size_t bh = (size_t)b * p.H + h;
  const int stride = 2 + p.r_v;
  const float* parts = p.partials + bh * p.S * stride;
  float m_s = -INFINITY, dot = 0.f;
  if (tid < p.S) m_s = __ldcg(parts + (size_t)tid * stride);
  for (int i = tid; i < p.d; i += 128) dot = fmaf(p.q[bh * p.d + i], p.k_self[bh * p.d + i], dot);
  const float mx = warp_max_f(m_s), ds = warp_sum_f(dot);
  if (lane == 0) {
    red[w] = mx;
    red[4 + w] = ds;
  }
  named_barrier(bar, 128);
  const float M_hist = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float s_self = p.kappa * ((red[4] + red[5]) + (red[6] + red[7]));
  const float M = fmaxf(M_hist, s_self);
  if (tid < p.S) wts[tid] = exp2f(m_s - M);
  named_barrier(bar, 128);
  // loads are issued in batches of 8 or 16 before they are used: from L2 under load
  // each round trip is long, and only a warpgroup runs this
  float l_hist = 0.f;
  for (int s0 = 0; s0 < p.S; s0 += 8) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = s0 + e < p.S ? __ldcg(parts + (size_t)(s0 + e) * stride + 1) : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) l_hist = fmaf(v[e], s0 + e < p.S ? wts[s0 + e] : 0.f, l_hist);
  }
  const float w_self = exp2f(s_self - M);
  const float inv = 1.f / (l_hist + w_self);
  for (int m = tid; m < p.r_v; m += 128) {
    float acc = 0.f;
    for (int s0 = 0; s0 < p.S; s0 += 8) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        v[e] = s0 + e < p.S ? __ldcg(parts + (size_t)(s0 + e) * stride + 2 + m) : 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(v[e], s0 + e < p.S ? wts[s0 + e] : 0.f, acc);
    }
    olat[m] = acc * inv;
  }
  named_barrier(bar, 128);
  if (tid < p.d) {
    // W_up,v,t,h packed transposed ([r_v][d]): the loads of consecutive threads coalesce
    const float* Wt = p.wupv_t + (size_t)h * p.d * p.r_v + tid;
    float y = 0.f;
    for (int m0 = 0; m0 < p.r_v; m0 += 16) {
      float wv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) wv[e] = m0 + e < p.r_v ? Wt[(size_t)(m0 + e) * p.d] : 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) y = fmaf(wv[e], m0 + e < p.r_v ? olat[m0 + e] : 0.f, y);
    }
    p.out[bh * p.d + tid] = y + (l_hist * inv) * p.muv_t[(size_t)h * p.d + tid] +
                            (w_self * inv) * p.v_self[bh * p.d + tid];
  }
  named_barrier(bar, 128);   // scratch is reused by the next head
}

// D: rotated dims per head.  NOPE (decoupled RoPE): each head's score operand has
// 16 more columns, the first of which is the NoPE content score (read by
// warpgroup 0 and added to the rotary branch's score).
template <int D, int G, bool FUSE, bool NOPE>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const __grid_constant__ TcParams p) {
  constexpr int NS = D + (NOPE ? 16 : 0);   // score columns per head
  constexpr int HALF = D / 2;
  constexpr int WG_PAIRS = HALF / kEpiWG;   // RoPE pairs per epilogue warpgroup
  constexpr int WG_COLS = 2 * WG_PAIRS;     // TMEM columns per warpgroup (Re, Im interleaved)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_k = reinterpret_cast<uint64_t*>(sm + p.bar_off);   // [nst] K latent tile landed
  uint64_t* empty_k = full_k + p.nst;                                // [nst] score MMA done with it
  uint64_t* full_v = empty_k + p.nst;                                // [nst_v] V latent tile landed
  uint64_t* empty_v = full_v + p.nst_v;                              // [nst_v] V MMA done with it
  uint64_t* tfull = empty_v + p.nst_v;   // [2] scores in TMEM
  uint64_t* tempty = tfull + 2;          // [2] scores read
  uint64_t* bfull = tempty + 2;          // [2] query-absorbed operands loaded
  uint64_t* bempty = bfull + 2;          // [2] operand buffer free
  uint64_t* pfull = bempty + 2;          // [2] softmax weights written
  uint64_t* pempty = pfull + 2;          // [2] V MMA done with the weights buffer
  uint64_t* drain = pempty + 2;          // [2] each MMA issuer's last MMAs completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + p.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + p.misc_off + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ops_head_bytes = p.b_head_bytes;
  const int* ctx_s = p.B <= kCtxCache ? reinterpret_cast<const int*>(sm + p.ctx_off) : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full_k[s], 1);
      mbar_init(&empty_k[s], 1);
    }
    for (int s = 0; s < p.nst_v; ++s) {
      mbar_init(&full_v[s], 1);
      mbar_init(&empty_v[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps);
      mbar_init(&bfull[a], 1);
      mbar_init(&bempty[a], 1);
      mbar_init(&pfull[a], 4);
      mbar_init(&pempty[a], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 2 + kEpiWarps) {
    const int et = threadIdx.x - 64;
    if (ctx_s) {
      int* cs = reinterpret_cast<int*>(sm + p.ctx_off);
      for (int b = et; b < p.B; b += kEpiThreads) {
        int n = p.ctx_len[b];
        if (n < 0 || n > p.n_cap) {
          if (blockIdx.x == 0) atomicOr(p.status, LLA_STATUS_CTX_RANGE);
          n = n < 0 ? 0 : p.n_cap;
        }
        cs[b] = n;
      }
    }
    if (et < 64) {
      reinterpret_cast<float2*>(sm + p.rope_off)[et] = p.step[et];
      reinterpret_cast<uint2*>(sm + p.rope_off + 512)[et] = make_uint2(p.phi_lo[et], p.phi_hi[et]);
    }
    // ones tile: one 8-row group (K columns 0 and 1 hold 1.0) that every row group aliases
    if (et < 8 * 16) {
      const int m = et / 16, k = et % 16;
      *reinterpret_cast<__nv_bfloat16*>(sm + p.ones_off + (k >> 3) * 128 + m * 16 + (k & 7) * 2) =
          __float2bfloat16_rn(k < 2 ? 1.f : 0.f);
    }
    // softmax-weight tiles (two buffers x G heads, 8 rows x 128 tokens): rows 2..7 stay 0
    for (int idx = et; idx < 2 * G * 8 * kTile / 2; idx += kEpiThreads)
      reinterpret_cast<uint32_t*>(sm + p.p_off)[idx] = 0u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == kVProdWarp) {
    // ------------------------------------------------------------ TMA producers
    // warp 0 streams the K latents (and each item's operand images), warp kVProdWarp
    // the V latents; each ring is released by the MMA that reads it.
    if (lane == 0) {
      const bool kside = warp == 0;
      const CUtensorMap* map = kside ? &map_k : &map_v;
      tma_prefetch_desc(map);
      const int nst = kside ? p.nst : p.nst_v;
      uint64_t* fullb = kside ? full_k : full_v;
      uint64_t* emptyb = kside ? empty_k : empty_v;
      uint32_t it = 0, jn = 0;
      RingPos rs;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        if (r.ntiles == 0) continue;
        if (kside) {
          // query-absorbed operands of this item into B buffer jn & 1 (written by the
          // prep grid, which may still be running when this kernel starts)
          if (jn == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
          const uint32_t buf = jn & 1u, bph = (jn >> 1) & 1u;
          if (!mbar_wait(&bempty[buf], bph ^ 1u, abort_flag)) break;
          const size_t head0 = (size_t)r.b * p.H + (size_t)r.hg * G;
          mbar_arrive_expect_tx(&bfull[buf], G * (ops_head_bytes + p.bias_head_bytes));
          bulk_load(sm + p.b_off + buf * G * ops_head_bytes, p.ops_b + head0 * ops_head_bytes,
                    G * ops_head_bytes, &bfull[buf]);
          bulk_load(sm + p.bias_off + buf * G * p.bias_head_bytes,
                    p.ops_bias + head0 * p.bias_head_bytes, G * p.bias_head_bytes, &bfull[buf]);
          ++jn;
        }
        for (int k = 0; k < r.ntiles; ++k, ++it, rs.next(nst)) {
          const uint32_t stage = rs.slot, ph = rs.phase;
          if (!mbar_wait(&emptyb[stage], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const int y = r.tok0 + k * kTile;
          if (kside) {
            mbar_arrive_expect_tx(&fullb[stage], p.tx_bytes);
            unsigned char* st = sm + p.st_off + stage * p.st_bytes;
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const int h = r.hg * G + g;
              for (int kb = 0; kb < p.nkb; ++kb)
                tma_load_3d(st + (g * p.nkb + kb) * p.box_bytes, map, &fullb[stage],
                            h * p.lat_hk + kb * p.box_k, y, r.b);
            }
          } else {
            mbar_arrive_expect_tx(&fullb[stage], p.tx_v);
            unsigned char* st = sm + p.stv_off + stage * p.stv_bytes;
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const int h = r.hg * G + g;
              for (int vb = 0; vb < p.nvb; ++vb)
                tma_load_3d(st + (g * p.nvb + vb) * p.vbox_bytes, map, &fullb[stage],
                            h * p.lat_hv + vb * p.cvb, y, r.b);
            }
          }
        }
      }
      if (*abort_flag) {
        // Drain: wait (bounded) for every copy this thread issued before leaving.
        const uint32_t n_out = it < (uint32_t)nst ? it : (uint32_t)nst;
        for (uint32_t j = 0; j < n_out; ++j) {
          const uint32_t i = it - 1 - j;
          const uint32_t stage = i % nst, ph = (i / nst) & 1u;
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&fullb[stage], ph) && global_timer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
        for (uint32_t j = 0; kside && j < 2 && j < jn; ++j) {
          const uint32_t i = jn - 1 - j;
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&bfull[i & 1u], (i >> 1) & 1u) &&
                 global_timer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ score MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NS);
      const uint32_t sbo_a = 16u * p.box_k;
      const uint64_t odesc = smem_desc(smem_addr(sm + p.ones_off), 128, 0, 0);   // rows alias
      uint32_t it = 0, jn = 0;
      RingPos rk, ra;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        if (r.ntiles == 0) continue;
        const uint32_t buf = jn & 1u, bph = (jn >> 1) & 1u;
        if (!mbar_wait(&bfull[buf], bph, abort_flag)) {
          ok = false;
          break;
        }
        ++jn;
        const uint32_t b_base = smem_addr(sm + p.b_off + buf * G * ops_head_bytes);
        const uint32_t bias_base = smem_addr(sm + p.bias_off + buf * G * p.bias_head_bytes);
        for (int k = 0; k < r.ntiles; ++k, ++it, rk.next(p.nst), ra.next(p.nacc)) {
          const uint32_t stage = rk.slot, ph = rk.phase;
          const uint32_t acc = ra.slot, aph = ra.phase;
          if (!mbar_wait(&full_k[stage], ph, abort_flag) ||
              !mbar_wait(&tempty[acc], aph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st_addr = smem_addr(sm + p.st_off + stage * p.st_bytes);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint32_t d_tmem = tmem_base + acc * p.acc_cols + g * NS;
            const uint32_t b_addr = b_base + g * ops_head_bytes;
            for (int kk = 0; kk < p.K_pad / 16; ++kk) {
              const int kb = (kk * 16) / p.box_k, kin = (kk * 16) % p.box_k;
              const uint64_t adesc =
                  smem_desc(st_addr + (g * p.nkb + kb) * p.box_bytes + kin * 2, 16, sbo_a, p.swz);
              const uint64_t bdesc = smem_desc(b_addr + kk * 256, 128, p.b_sbo, 0);
              mma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
            }
            const uint64_t bias_desc = smem_desc(bias_base + g * p.bias_head_bytes, 128, 256, 0);
            mma_bf16(d_tmem, odesc, bias_desc, idesc, 1u);
          }
          mma_commit(&tfull[acc]);
          mma_commit(&empty_k[stage]);
          if (k == r.ntiles - 1) mma_commit(&bempty[buf]);   // last use of this B buffer
        }
      }
      mma_drain(&drain[0]);
    }
    __syncwarp();
  } else if (warp == kVMmaWarp) {
    // ------------------------------------------------------------ V MMA issuer
    // D_v[g] (+)= P_i[g] (rows 0, 1: weights hi, lo; all 8-row groups alias) x C_v,i[g]
    // (128 tokens x N_v latent dims, MN-major): one K=16 MMA per 16 tokens.
    if (lane == 0) {
      const uint32_t idesc_v = idesc_bf16_f32(128, p.N_v) | (1u << 16);   // B (c_v) MN-major
      const uint32_t sbo_v = 16u * p.cvb;          // 8 token rows of one MN box
      const uint32_t p_base = smem_addr(sm + p.p_off);
      uint32_t it = 0;
      RingPos rv;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        for (int k = 0; k < r.ntiles; ++k, ++it, rv.next(p.nst_v)) {
          const uint32_t pb = it & 1u;
          const uint32_t vs = rv.slot, vph = rv.phase;
          if (!mbar_wait(&pfull[pb], (it >> 1) & 1u, abort_flag) ||
              !mbar_wait(&full_v[vs], vph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t cv_addr = smem_addr(sm + p.stv_off + vs * p.stv_bytes);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const uint32_t d_tmem = tmem_base + p.v_col0 + g * p.N_v;
            const uint32_t a_addr = p_base + (pb * G + g) * (8 * kTile * 2);
            const uint32_t b_addr = cv_addr + g * p.nvb * p.vbox_bytes;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t adesc = smem_desc(a_addr + kk * 256, 128, 0, 0);
              const uint64_t bdesc =
                  smem_desc(b_addr + kk * 2 * sbo_v, p.vbox_bytes, sbo_v, p.swz_v);
              mma_bf16(d_tmem, adesc, bdesc, idesc_v, (k == 0 && kk == 0) ? 0u : 1u);
            }
          }
          mma_commit(&pempty[pb]);
          mma_commit(&empty_v[vs]);
        }
      }
      mma_drain(&drain[1]);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;
    const int wgi = (warp - 2) >> 2;          // which part of the RoPE pairs
    const int sub = warp & 3;                 // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;          // token row of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
    float* sbuf = reinterpret_cast<float*>(sm + p.sbuf_off);   // [2][kEpiWG - 1][G][128]
    float* red = reinterpret_cast<float*>(sm + p.red_off);     // [G][4]

    TileCursor pc;
    cursor_first(p, ctx_s, pc);
    // conj(e^{i p theta_i}) for this thread's RoPE pairs at position pos_cur of its
    // token; when the next tile's token sits exactly one tile further on, the
    // factors advance by one complex product, otherwise they are recomputed.
    float2 ef[WG_PAIRS];
    int pos_cur = kNoPos, run = 0;
    const float2* step_s = reinterpret_cast<const float2*>(sm + p.rope_off) + wgi * WG_PAIRS;
    const uint2* phi_s = reinterpret_cast<const uint2*>(sm + p.rope_off + 512) + wgi * WG_PAIRS;
    auto advance_rope = [&](int praw) {
      if (praw == kNoPos) return;               // row past the context: keep factors
      const int pn = checked_pos(p, praw);
      if (pos_cur != kNoPos && pn == pos_cur + kTile && run < kReseedTiles) {
#pragma unroll
        for (int q = 0; q < WG_PAIRS; ++q) {
          const float2 st = step_s[q];
          const float2 e = ef[q];
          ef[q] = make_float2(fmaf(e.x, st.x, -e.y * st.y), fmaf(e.x, st.y, e.y * st.x));
        }
        ++run;
      } else {
#pragma unroll
        for (int q = 0; q < WG_PAIRS; ++q) {
          const uint2 ph = phi_s[q];
          ef[q] = rope_factor(static_cast<uint32_t>(pn), ph.x, ph.y);
        }
        run = 0;
      }
      pos_cur = pn;
    };
#pragma unroll
    for (int q = 0; q < WG_PAIRS; ++q) ef[q] = make_float2(1.f, 0.f);
    advance_rope(cursor_pos(p, pc, row));
    cursor_next(p, ctx_s, pc);
    int pos_next = cursor_pos(p, pc, row);
    cursor_next(p, ctx_s, pc);

    uint32_t it = 0;
    RingPos ra;
    bool aborted = false;
    for (int item = blockIdx.x; !aborted && item < p.n_items; item += gridDim.x) {
      const ItemRange r = item_range(p, ctx_s, item, et == 0 && !ctx_s);
      float m_ref[G], l_part[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m_ref[g] = -INFINITY;
        l_part[g] = 0.f;
      }
      // fused finish, set up while the tiles stream: the in-flight scores' partial
      // dot products q . k_self go to shared memory (per warp of warpgroup 0), and the
      // heads' W_up,v rows into L2, kept there ahead of the latent stream
      if constexpr (FUSE) {
        float* misc = reinterpret_cast<float*>(sm + p.comb_off) + 512;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const size_t bh = (size_t)r.b * p.H + r.hg * G + g;
          if (wgi == 0) {
            const float qk = row < p.d ? __ldg(p.q + bh * p.d + row) * __ldg(p.k_self + bh * p.d + row) : 0.f;
            const float sdot = warp_sum_f(qk);
            if (lane == 0) misc[8 + g * 4 + sub] = sdot;
          }
          const char* wrow = reinterpret_cast<const char*>(p.wupv_t + (size_t)(r.hg * G + g) * p.d * p.r_v);
          for (int off = et * 128; off < p.d * p.r_v * 4; off += kEpiThreads * 128)
            asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(wrow + off));
        }
      }
      for (int k = 0; k < r.ntiles; ++k, ++it, ra.next(p.nacc)) {
        const uint32_t acc = ra.slot, aph = ra.phase;
        const int t0 = r.tok0 + k * kTile;
        const int cnt = min(kTile, r.tok_end - t0);
        const bool valid = row < cnt;

        bool ok = mbar_wait(&tfull[acc], aph, abort_flag);
        tc_fence_after();
        float part[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint32_t head_col = tmem_base + lane_addr + acc * p.acc_cols + g * NS;
          const uint32_t col = head_col + wgi * WG_COLS;
          float u[WG_COLS];
#pragma unroll
          for (int c = 0; c < WG_COLS / 16; ++c) tmem_ld16(col + c * 16, u + c * 16);
          if constexpr (WG_COLS % 16 != 0) tmem_ld8(col + (WG_COLS / 16) * 16, u + (WG_COLS / 16) * 16);
          float un[8];
          un[0] = 0.f;
          if constexpr (NOPE) {
            if (wgi == 0) tmem_ld8(head_col + D, un);   // the NoPE content column (+ 7 zeros)
          }
          tmem_wait_ld();
          float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int q = 0; q < WG_PAIRS; q += 2) {
            a0 = ffma2(make_float2(u[2 * q], u[2 * q + 1]), ef[q], a0);
            if (q + 1 < WG_PAIRS) a1 = ffma2(make_float2(u[2 * q + 2], u[2 * q + 3]), ef[q + 1], a1);
          }
          part[g] = (a0.x + a0.y) + (a1.x + a1.y) + un[0];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        if (wgi > 0) {
#pragma unroll
          for (int g = 0; g < G; ++g)
            sbuf[(((it & 1u) * (kEpiWG - 1) + (wgi - 1)) * G + g) * kTile + row] = part[g];
        }
        if (epi_barrier_or(!ok)) {
          aborted = true;
          break;
        }
        if (wgi == 0) {
          // ---- softmax weights against the item's reference maximum m_ref, taken on
          // the item's first tile; later tiles only check (one barrier) that no score
          // exceeds it by more than 2^kRescaleLog2, and take a new maximum if one does
          float s[G];
          int over = 0;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float tot = part[g];
#pragma unroll
            for (int w = 0; w < kEpiWG - 1; ++w)
              tot += sbuf[(((it & 1u) * (kEpiWG - 1) + w) * G + g) * kTile + row];
            s[g] = valid ? tot : -INFINITY;
            over |= s[g] > m_ref[g] + kRescaleLog2;
          }
          bool rescale = false;
          float alpha[G];
#pragma unroll
          for (int g = 0; g < G; ++g) alpha[g] = 1.f;
          if (k == 0 || wg_barrier_or(2, over)) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float mx = warp_max_f(s[g]);
              if (lane == 0) red[g * 4 + sub] = mx;
            }
            named_barrier(2, 128);
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float mt =
                  fmaxf(fmaxf(red[g * 4], red[g * 4 + 1]), fmaxf(red[g * 4 + 2], red[g * 4 + 3]));
              if (k == 0) {
                m_ref[g] = mt;
              } else if (mt > m_ref[g] + kRescaleLog2) {
                alpha[g] = exp2f(m_ref[g] - mt);
                m_ref[g] = mt;
                rescale = true;
              }
            }
            named_barrier(2, 128);   // every warp has read red before it is reused
          }
          const uint32_t pb = it & 1u;
          // the weights buffer is free once the V MMA of tile it - 2 has finished
          ok = mbar_wait(&pempty[pb], ((it >> 1) & 1u) ^ 1u, abort_flag);
          if (rescale) {
            // rare: rescale the item's V accumulator (TMEM lanes 0 and 1) once the V MMA
            // of the previous tile has finished; sub-partition 0 (lanes 0-31) does it
            ok = ok && mbar_wait(&pempty[(it - 1) & 1u], ((it - 1) >> 1) & 1u, abort_flag);
            tc_fence_after();
            if (sub == 0) {
#pragma unroll
              for (int g = 0; g < G; ++g) {
                for (int c = 0; c < p.N_v; c += 16) {
                  float v[16];
                  const uint32_t ta = tmem_base + p.v_col0 + g * p.N_v + c;
                  tmem_ld16(ta, v);
                  tmem_wait_ld();
#pragma unroll
                  for (int e = 0; e < 16; ++e) v[e] *= alpha[g];
                  tmem_st16(ta, v);
                }
              }
              tmem_wait_st();
            }
            tc_fence_before();
          }
          if (cnt < kTile) {
            // rows past the context: zero them in the V stage, so that the V MMA takes
            // zero weights times zeros whatever the cache holds there
            const uint32_t vs = it % p.nst_v, vph = (it / p.nst_v) & 1u;   // partial tiles only
            ok = ok && mbar_wait(&full_v[vs], vph, abort_flag);
            if (!valid) {
              const uint32_t rbytes = (uint32_t)p.cvb * 2;                 // bytes of a box row
              unsigned char* vrow = sm + p.stv_off + vs * p.stv_bytes + row * rbytes;
              for (int bx = 0; bx < G * p.nvb; ++bx)
                for (uint32_t c = 0; c < rbytes; c += 16)
                  *reinterpret_cast<uint4*>(vrow + bx * p.vbox_bytes + c) = make_uint4(0, 0, 0, 0);
            }
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pj = valid ? exp2f(s[g] - m_ref[g]) : 0.f;
            l_part[g] = l_part[g] * alpha[g] + pj;
            const __nv_bfloat16 hi = __float2bfloat16_rn(pj);
            const __nv_bfloat16 lo = __float2bfloat16_rn(pj - __bfloat162float(hi));
            unsigned char* pt = sm + p.p_off + (pb * G + g) * (8 * kTile * 2) +
                                (row >> 3) * 128 + (row & 7) * 2;
            *reinterpret_cast<__nv_bfloat16*>(pt) = hi;
            *reinterpret_cast<__nv_bfloat16*>(pt + 16) = lo;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pfull[pb]);   // one arrival per warp of the group
        }
        if (!ok) *abort_flag = 1;
        // off the critical path: RoPE factors of the next tile (its position was
        // loaded a tile ago) and the raw position of the tile after it
        advance_rope(pos_next);
        pos_next = cursor_pos(p, pc, row);
        cursor_next(p, ctx_s, pc);
      }
      if (aborted) break;
      // ---------------------------------------------------------- item partial
      if constexpr (FUSE) {
        // One split per group: finish its heads here from on-chip state with both
        // warpgroups: o = (W_up,v o_lat a + mu_v l a + v_self b) / (l a + b), where
        // a = 2^(m - M), b = 2^(s_self - M), M = max(m, s_self) (base-2 scores).
        float* olat = reinterpret_cast<float*>(sm + p.comb_off);   // [r_v]
        float* yh = olat + 256;                                      // [2][128]
        float* misc = yh + 256;             // [32]: m per head [0, 4), q . k_self partials [8, 24)
        if (wgi == 0) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float l = warp_sum_f(l_part[g]);
            if (lane == 0) red[g * 4 + sub] = l;
            if (row == 0) misc[g] = m_ref[g];
          }
        }
        bool okv = true;
        if (wgi == 0 && r.ntiles > 0) {
          const uint32_t last = it - 1;
          okv = __all_sync(0xffffffffu, mbar_wait(&pempty[last & 1u], (last >> 1) & 1u, abort_flag));
          tc_fence_after();
        }
        for (int g = 0; g < G; ++g) {
          named_barrier(1, kEpiThreads);            // red, misc visible; scratch free
          if (wgi == 0 && sub == 0) {
            // V accumulator lanes 0 (hi) and 1 (lo) of head g -> olat
            if (r.ntiles > 0 && okv) {
              for (int c = 0; c < p.N_v; c += 16) {
                float v[16];
                tmem_ld16(tmem_base + p.v_col0 + g * p.N_v + c, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const float o = v[e] + __shfl_down_sync(0xffffffffu, v[e], 1);
                  if (lane == 0 && c + e < p.r_v) olat[c + e] = o;
                }
              }
            } else {
              for (int m = lane; m < p.r_v; m += 32) olat[m] = 0.f;
            }
          }
          named_barrier(1, kEpiThreads);            // olat complete
          const float m_h = r.ntiles > 0 ? misc[g] : -INFINITY;
          const float l_h = (red[g * 4] + red[g * 4 + 1]) + (red[g * 4 + 2] + red[g * 4 + 3]);
          const float s_self =
              p.kappa * ((misc[8 + g * 4] + misc[8 + g * 4 + 1]) + (misc[8 + g * 4 + 2] + misc[8 + g * 4 + 3]));
          const float M = fmaxf(m_h, s_self);
          const float a = r.ntiles > 0 ? exp2f(m_h - M) : 0.f, bsf = exp2f(s_self - M);
          const float inv = 1.f / (l_h * a + bsf);
          // up-projection: warpgroup hf sums half of the latent dims for output dim d_i
          const int d_i = et & 127, hf = et >> 7;
          const int half_r = (p.r_v + 1) / 2, m0 = hf * half_r, m1 = min(p.r_v, m0 + half_r);
          const size_t bh = (size_t)r.b * p.H + r.hg * G + g;
          float vs_d = 0.f, mu_d = 0.f;
          if (hf == 0 && d_i < p.d) {
            vs_d = __ldg(p.v_self + bh * p.d + d_i);
            mu_d = __ldg(p.muv_t + (size_t)(r.hg * G + g) * p.d + d_i);
          }
          float y = 0.f;
          if (d_i < p.d) {
            const float* Wt = p.wupv_t + (size_t)(r.hg * G + g) * p.d * p.r_v + d_i;
            for (int mb = m0; mb < m1; mb += 16) {
              float wv[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) wv[e] = mb + e < m1 ? __ldg(Wt + (size_t)(mb + e) * p.d) : 0.f;
#pragma unroll
              for (int e = 0; e < 16; ++e) y = fmaf(wv[e], mb + e < m1 ? olat[mb + e] : 0.f, y);
            }
          }
          yh[hf * 128 + d_i] = y;
          named_barrier(1, kEpiThreads);            // both halves written
          if (hf == 0 && d_i < p.d)
            p.out[bh * p.d + d_i] = ((yh[d_i] + yh[128 + d_i]) * a + mu_d * (l_h * a) + vs_d * bsf) * inv;
        }
        named_barrier(1, kEpiThreads);              // scratch free for the next item
      } else if (wgi == 0 && r.ntiles > 0) {
        const size_t bh0 = (size_t)r.b * p.H + r.hg * G;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float l = warp_sum_f(l_part[g]);
          if (lane == 0) red[g * 4 + sub] = l;
        }
        // V accumulator: wait for the item's last V MMA, then read lanes 0 (hi) and 1 (lo)
        const uint32_t last = it - 1;
        const bool okv =
            __all_sync(0xffffffffu, mbar_wait(&pempty[last & 1u], (last >> 1) & 1u, abort_flag));
        tc_fence_after();
        named_barrier(2, 128);
        if (sub == 0 && okv) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float* part_out = p.partials + ((bh0 + g) * p.S + r.s) * (2 + p.r_v);
            if (lane == 0) {
              part_out[0] = m_ref[g];
              part_out[1] = red[g * 4] + red[g * 4 + 1] + red[g * 4 + 2] + red[g * 4 + 3];
            }
            for (int c = 0; c < p.N_v; c += 16) {
              float v[16];
              tmem_ld16(tmem_base + p.v_col0 + g * p.N_v + c, v);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float o = v[e] + __shfl_down_sync(0xffffffffu, v[e], 1);
                if (lane == 0 && c + e < p.r_v) part_out[2 + c + e] = o;
              }
            }
          }
        }
        tc_fence_before();
        named_barrier(2, 128);
      } else if (wgi == 0 && !FUSE) {
        // no tiles in this split: empty partial
        const size_t bh0 = (size_t)r.b * p.H + r.hg * G;
        for (int idx = row; idx < G * (2 + p.r_v); idx += 128) {
          const int g = idx / (2 + p.r_v), m = idx % (2 + p.r_v);
          p.partials[((bh0 + g) * p.S + r.s) * (2 + p.r_v) + m] = m == 0 ? -INFINITY : 0.f;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
  if (threadIdx.x == 0) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // prep's counter and status writes
    if (*abort_flag) atomicOr(p.status, LLA_STATUS_TIMEOUT);
    if constexpr (FUSE) {
      // with the combine fused in, the last CTA to finish publishes this call's status
      // bits (word 1) and clears word 0; otherwise the combine pass does it
      __threadfence();
      if (atomicAdd(&p.counters[(size_t)p.B * p.H], 1u) == gridDim.x - 1) {
        __threadfence();
        p.status[1] = atomicExch(&p.status[0], 0);
      }
    }
  }
}

// LLA-2D: every head reads the same latent row (close reading §二.6), so a work
// item (sequence b, group of HP heads, context split s) streams each 128-token
// c_k and c_v tile once and uses it for all HP heads:
//   * warp 1 issues the score MMAs head by head, U_h = C_k A~_h^T (+ bias), each
//     into the next of nacc one-head TMEM buffers, so the epilogue drains head h
//     while head h + 1 is multiplied;
//   * warp 11 sums V transposed, D_v^T[r_v x 2 HP] += C_v^T P^T: the staged c_v
//     tile is the MN-major A operand (M = 128 latent dims per block) and the
//     softmax weights of all HP heads (rows 2g: hi, 2g + 1: lo) are the K-major
//     B operand, so one set of K = 16 MMAs per tile serves the whole group.
// The epilogue has four warpgroups, each owning a quarter of the RoPE pairs of
// every token row (so a thread keeps 16 complex factors and the TMEM reads of a
// head spread over 16 warps); warpgroup g also finalizes head g of the group:
// its softmax, its weight rows, rescales and its partial.  Producers, bounded
// waits and the abort path are those of decode_tc_kernel.
constexpr int kEpiWG2 = 4;
constexpr int kEpiThreads2 = 128 * kEpiWG2;
constexpr int kEpiWarps2 = kEpiThreads2 / 32;
constexpr int kThreads2 = 64 + kEpiThreads2 + 64;
constexpr int kVProdWarp2 = 2 + kEpiWarps2, kVMmaWarp2 = 3 + kEpiWarps2;

template <int D, int HP, bool FUSE, bool NOPE>
__global__ void __launch_bounds__(kThreads2, 1)
    decode_tc2d_kernel(const __grid_constant__ CUtensorMap map_k,
                       const __grid_constant__ CUtensorMap map_v, const __grid_constant__ TcParams p) {
  constexpr int NS = D + (NOPE ? 16 : 0);   // score columns per head (see decode_tc_kernel)
  constexpr int HALF = D / 2;
  constexpr int WG_PAIRS = HALF / kEpiWG2;
  static_assert(HP <= kEpiWG2, "one finalizing warpgroup per head");
  constexpr int WG_COLS = 2 * WG_PAIRS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_k = reinterpret_cast<uint64_t*>(sm + p.bar_off);   // [nst]
  uint64_t* empty_k = full_k + p.nst;                                // [nst]
  uint64_t* full_v = empty_k + p.nst;                                // [nst_v]
  uint64_t* empty_v = full_v + p.nst_v;                              // [nst_v]
  uint64_t* tfull = empty_v + p.nst_v;   // [nacc] one head's scores in TMEM
  uint64_t* tempty = tfull + 4;          // [nacc] scores read
  uint64_t* bfull = tempty + 4;          // [nbuf_b] query-absorbed operands loaded
  uint64_t* bempty = bfull + 2;          // [nbuf_b] operand buffer free
  uint64_t* pfull = bempty + 2;          // [2] softmax weights written
  uint64_t* pempty = pfull + 2;          // [2] V MMA done with the weights buffer
  uint64_t* drain = pempty + 2;          // [2] each MMA issuer's last MMAs completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + p.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + p.misc_off + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ops_head_bytes = p.b_head_bytes;
  const int* ctx_s = p.B <= kCtxCache ? reinterpret_cast<const int*>(sm + p.ctx_off) : nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full_k[s], 1);
      mbar_init(&empty_k[s], 1);
    }
    for (int s = 0; s < p.nst_v; ++s) {
      mbar_init(&full_v[s], 1);
      mbar_init(&empty_v[s], 1);
    }
    for (int a = 0; a < p.nacc; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarps2);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bfull[a], 1);
      mbar_init(&bempty[a], 1);
      mbar_init(&pfull[a], 4 * HP);
      mbar_init(&pempty[a], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 2 + kEpiWarps2) {
    const int et = threadIdx.x - 64;
    if (ctx_s) {
      int* cs = reinterpret_cast<int*>(sm + p.ctx_off);
      for (int b = et; b < p.B; b += kEpiThreads2) {
        int n = p.ctx_len[b];
        if (n < 0 || n > p.n_cap) {
          if (blockIdx.x == 0) atomicOr(p.status, LLA_STATUS_CTX_RANGE);
          n = n < 0 ? 0 : p.n_cap;
        }
        cs[b] = n;
      }
    }
    if (et < 64) {
      reinterpret_cast<float2*>(sm + p.rope_off)[et] = p.step[et];
      reinterpret_cast<uint2*>(sm + p.rope_off + 512)[et] = make_uint2(p.phi_lo[et], p.phi_hi[et]);
    }
    if (et < 8 * 16) {
      const int m = et / 16, k = et % 16;
      *reinterpret_cast<__nv_bfloat16*>(sm + p.ones_off + (k >> 3) * 128 + m * 16 + (k & 7) * 2) =
          __float2bfloat16_rn(k < 2 ? 1.f : 0.f);
    }
    // both weight buffers start zero: rows >= 2 HP are never written
    for (int idx = et; idx < 2 * (int)p.p_buf_bytes / 4; idx += kEpiThreads2)
      reinterpret_cast<uint32_t*>(sm + p.p_off)[idx] = 0u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == kVProdWarp2) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool kside = warp == 0;
      const CUtensorMap* map = kside ? &map_k : &map_v;
      tma_prefetch_desc(map);
      const int nst = kside ? p.nst : p.nst_v;
      uint64_t* fullb = kside ? full_k : full_v;
      uint64_t* emptyb = kside ? empty_k : empty_v;
      uint32_t it = 0, jn = 0;
      RingPos rs;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        if (r.ntiles == 0) continue;
        if (kside) {
          const uint32_t buf = jn % p.nbuf_b, bph = (jn / p.nbuf_b) & 1u;
          if (!mbar_wait(&bempty[buf], bph ^ 1u, abort_flag)) break;
          const size_t head0 = (size_t)r.b * p.H + (size_t)r.hg * HP;
          mbar_arrive_expect_tx(&bfull[buf], HP * (ops_head_bytes + p.bias_head_bytes));
          bulk_load(sm + p.b_off + buf * HP * ops_head_bytes, p.ops_b + head0 * ops_head_bytes,
                    HP * ops_head_bytes, &bfull[buf]);
          bulk_load(sm + p.bias_off + buf * HP * p.bias_head_bytes,
                    p.ops_bias + head0 * p.bias_head_bytes, HP * p.bias_head_bytes, &bfull[buf]);
          ++jn;
        }
        for (int k = 0; k < r.ntiles; ++k, ++it, rs.next(nst)) {
          const uint32_t stage = rs.slot, ph = rs.phase;
          if (!mbar_wait(&emptyb[stage], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const int y = r.tok0 + k * kTile;
          if (kside) {
            mbar_arrive_expect_tx(&fullb[stage], p.tx_bytes);
            unsigned char* st = sm + p.st_off + stage * p.st_bytes;
            for (int kb = 0; kb < p.nkb; ++kb)
              tma_load_3d(st + kb * p.box_bytes, map, &fullb[stage], kb * p.box_k, y, r.b);
          } else {
            mbar_arrive_expect_tx(&fullb[stage], p.tx_v);
            unsigned char* st = sm + p.stv_off + stage * p.stv_bytes;
            for (int vb = 0; vb < p.nvb; ++vb)
              tma_load_3d(st + vb * p.vbox_bytes, map, &fullb[stage], vb * p.cvb, y, r.b);
          }
        }
      }
      if (*abort_flag) {
        const uint32_t n_out = it < (uint32_t)nst ? it : (uint32_t)nst;
        for (uint32_t j = 0; j < n_out; ++j) {
          const uint32_t i = it - 1 - j;
          const uint32_t stage = i % nst, ph = (i / nst) & 1u;
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&fullb[stage], ph) && global_timer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
        for (uint32_t j = 0; kside && j < (uint32_t)p.nbuf_b && j < jn; ++j) {
          const uint32_t i = jn - 1 - j;
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&bfull[i % p.nbuf_b], (i / p.nbuf_b) & 1u) &&
                 global_timer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ score MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NS);
      const uint32_t sbo_a = 16u * p.box_k;
      const uint64_t odesc = smem_desc(smem_addr(sm + p.ones_off), 128, 0, 0);   // rows alias
      uint32_t it = 0, jn = 0;
      RingPos rk, ra;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        if (r.ntiles == 0) continue;
        const uint32_t buf = jn % p.nbuf_b, bph = (jn / p.nbuf_b) & 1u;
        if (!mbar_wait(&bfull[buf], bph, abort_flag)) {
          ok = false;
          break;
        }
        ++jn;
        const uint32_t b_base = smem_addr(sm + p.b_off + buf * HP * ops_head_bytes);
        const uint32_t bias_base = smem_addr(sm + p.bias_off + buf * HP * p.bias_head_bytes);
        for (int k = 0; ok && k < r.ntiles; ++k, ++it, rk.next(p.nst)) {
          const uint32_t stage = rk.slot, ph = rk.phase;
          if (!mbar_wait(&full_k[stage], ph, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st_addr = smem_addr(sm + p.st_off + stage * p.st_bytes);
#pragma unroll 1
          for (int g = 0; g < HP; ++g, ra.next(p.nacc)) {
            const uint32_t acc = ra.slot, aph = ra.phase;
            if (!(p.poll ? mbar_wait_poll(&tempty[acc], aph ^ 1u, abort_flag)
                         : mbar_wait(&tempty[acc], aph ^ 1u, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * NS;
            const uint32_t b_addr = b_base + g * ops_head_bytes;
            for (int kk = 0; kk < p.K_pad / 16; ++kk) {
              const int kb = (kk * 16) / p.box_k, kin = (kk * 16) % p.box_k;
              const uint64_t adesc =
                  smem_desc(st_addr + kb * p.box_bytes + kin * 2, 16, sbo_a, p.swz);
              const uint64_t bdesc = smem_desc(b_addr + kk * 256, 128, p.b_sbo, 0);
              mma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
            }
            const uint64_t bias_desc = smem_desc(bias_base + g * p.bias_head_bytes, 128, 256, 0);
            mma_bf16(d_tmem, odesc, bias_desc, idesc, 1u);
            mma_commit(&tfull[acc]);
          }
          if (!ok) break;
          mma_commit(&empty_k[stage]);
          if (k == r.ntiles - 1) mma_commit(&bempty[buf]);   // last use of this B buffer
        }
      }
      mma_drain(&drain[0]);
    }
    __syncwarp();
  } else if (warp == kVMmaWarp2) {
    // ------------------------------------------------------------ V MMA issuer
    // D_v^T[block mb] (+)= C_v^T (128 latent dims x 128 tokens, MN-major A) x P^T
    // (128 tokens x n_p weight rows, K-major B): one K=16 MMA per 16 tokens.
    if (lane == 0) {
      const uint32_t idesc_v = idesc_bf16_f32(128, p.n_p) | (1u << 15);   // A (c_v) MN-major
      const uint32_t sbo_v = 16u * p.cvb;          // 8 token rows of one MN box
      const uint32_t boxes_per_block = 128u / p.cvb;
      const uint32_t p_base = smem_addr(sm + p.p_off);
      uint32_t it = 0;
      RingPos rv;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        for (int k = 0; k < r.ntiles; ++k, ++it, rv.next(p.nst_v)) {
          const uint32_t pb = it & 1u;
          const uint32_t vs = rv.slot, vph = rv.phase;
          if (!mbar_wait(&pfull[pb], (it >> 1) & 1u, abort_flag) ||
              !mbar_wait(&full_v[vs], vph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t cv_addr = smem_addr(sm + p.stv_off + vs * p.stv_bytes);
          const uint32_t b_addr = p_base + pb * p.p_buf_bytes;
          for (int mb = 0; mb < p.m_v; ++mb) {
            const uint32_t d_tmem = tmem_base + p.v_col0 + mb * p.n_p;
            const uint32_t a_addr = cv_addr + mb * boxes_per_block * p.vbox_bytes;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t adesc =
                  smem_desc(a_addr + kk * 2 * sbo_v, p.vbox_bytes, sbo_v, p.swz_v);
              const uint64_t bdesc = smem_desc(b_addr + kk * 256, 128, 2048, 0);
              mma_bf16(d_tmem, adesc, bdesc, idesc_v, (k == 0 && kk == 0) ? 0u : 1u);
            }
          }
          mma_commit(&pempty[pb]);
          mma_commit(&empty_v[vs]);
        }
      }
      mma_drain(&drain[1]);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;
    const int wgi = (warp - 2) >> 2;          // quarter of the RoPE pairs; head it finalizes
    const int sub = warp & 3;                 // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;          // token row of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
    const bool fin = wgi < HP;                // this warpgroup finalizes head wgi
    float* sbuf = reinterpret_cast<float*>(sm + p.sbuf_off);   // [2][HP][kEpiWG2][128]
    float* red = reinterpret_cast<float*>(sm + p.red_off);     // [HP][4]

    TileCursor pc;
    cursor_first(p, ctx_s, pc);
    float2 ef[WG_PAIRS];
    int pos_cur = kNoPos, run = 0;
    const float2* step_s = reinterpret_cast<const float2*>(sm + p.rope_off) + wgi * WG_PAIRS;
    const uint2* phi_s = reinterpret_cast<const uint2*>(sm + p.rope_off + 512) + wgi * WG_PAIRS;
    auto advance_rope = [&](int praw) {
      if (praw == kNoPos) return;
      const int pn = checked_pos(p, praw);
      if (pos_cur != kNoPos && pn == pos_cur + kTile && run < kReseedTiles) {
#pragma unroll
        for (int q = 0; q < WG_PAIRS; ++q) {
          const float2 st = step_s[q];
          const float2 e = ef[q];
          ef[q] = make_float2(fmaf(e.x, st.x, -e.y * st.y), fmaf(e.x, st.y, e.y * st.x));
        }
        ++run;
      } else {
#pragma unroll
        for (int q = 0; q < WG_PAIRS; ++q) {
          const uint2 ph = phi_s[q];
          ef[q] = rope_factor(static_cast<uint32_t>(pn), ph.x, ph.y);
        }
        run = 0;
      }
      pos_cur = pn;
    };
#pragma unroll
    for (int q = 0; q < WG_PAIRS; ++q) ef[q] = make_float2(1.f, 0.f);
    advance_rope(cursor_pos(p, pc, row));
    cursor_next(p, ctx_s, pc);
    int pos_next = cursor_pos(p, pc, row);
    cursor_next(p, ctx_s, pc);

    uint32_t it = 0;
    RingPos ra;
    bool aborted = false;
    for (int item = blockIdx.x; !aborted && item < p.n_items; item += gridDim.x) {
      const ItemRange r = item_range(p, ctx_s, item, et == 0 && !ctx_s);
      float m_ref = -INFINITY, l_part = 0.f;  // head wgi of the group (finalizing warpgroups)
      for (int k = 0; k < r.ntiles; ++k, ++it) {
        const int t0 = r.tok0 + k * kTile;
        const int cnt = min(kTile, r.tok_end - t0);
        const bool valid = row < cnt;
        const uint32_t par = it & 1u;
        bool ok = true;
#pragma unroll 1
        for (int g = 0; g < HP; ++g, ra.next(p.nacc)) {
          const uint32_t acc = ra.slot, aph = ra.phase;
          ok = ok && (p.poll ? mbar_wait_poll(&tfull[acc], aph, abort_flag)
                             : mbar_wait(&tfull[acc], aph, abort_flag));
          tc_fence_after();
          float uu[WG_COLS];
          const uint32_t col = tmem_base + lane_addr + acc * NS + wgi * WG_COLS;
#pragma unroll
          for (int c = 0; c < WG_COLS / 16; ++c) tmem_ld16(col + c * 16, uu + c * 16);
          if constexpr (WG_COLS % 16 != 0)
            tmem_ld8(col + (WG_COLS / 16) * 16, uu + (WG_COLS / 16) * 16);
          float un[8];
          un[0] = 0.f;
          if constexpr (NOPE) {
            if (wgi == 0) tmem_ld8(tmem_base + lane_addr + acc * NS + D, un);   // NoPE content column
          }
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
          float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int q = 0; q < WG_PAIRS; q += 2) {
            a0 = ffma2(make_float2(uu[2 * q], uu[2 * q + 1]), ef[q], a0);
            if (q + 1 < WG_PAIRS) a1 = ffma2(make_float2(uu[2 * q + 2], uu[2 * q + 3]), ef[q + 1], a1);
          }
          sbuf[((par * HP + g) * kEpiWG2 + wgi) * kTile + row] = (a0.x + a0.y) + (a1.x + a1.y) + un[0];
        }
        if (epi_barrier_or_n<kEpiThreads2>(!ok)) {
          aborted = true;
          break;
        }
        if (fin) {
          // ---- softmax weights of head wgi against the item's reference maximum
          const int g = wgi;
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < kEpiWG2; ++w) tot += sbuf[((par * HP + g) * kEpiWG2 + w) * kTile + row];
          const float sc = valid ? tot : -INFINITY;
          float alpha = 1.f;
          bool rescale = false;
          // reference maximum on the item's first tile; later tiles take a new one only
          // when a score exceeds it by more than 2^kRescaleLog2 (one barrier to check)
          if (k == 0 || wg_barrier_or(2 + wgi, sc > m_ref + kRescaleLog2)) {
            const float mx = warp_max_f(sc);
            if (lane == 0) red[g * 4 + sub] = mx;
            named_barrier(2 + wgi, 128);
            const float mt =
                fmaxf(fmaxf(red[g * 4], red[g * 4 + 1]), fmaxf(red[g * 4 + 2], red[g * 4 + 3]));
            if (k == 0) {
              m_ref = mt;
            } else if (mt > m_ref + kRescaleLog2) {
              alpha = exp2f(m_ref - mt);
              m_ref = mt;
              rescale = true;
            }
            named_barrier(2 + wgi, 128);
          }
          const uint32_t pb = it & 1u;
          // the weights buffer is free once the V MMA of tile it - 2 has finished
          ok = mbar_wait(&pempty[pb], ((it >> 1) & 1u) ^ 1u, abort_flag);
          if (rescale) {
            // rare: rescale head g's V accumulator columns 2g, 2g + 1 in every lane once
            // the V MMA of the previous tile has finished; each warp owns its 32 lanes
            ok = ok && mbar_wait(&pempty[(it - 1) & 1u], ((it - 1) >> 1) & 1u, abort_flag);
            tc_fence_after();
            for (int mb = 0; mb < p.m_v; ++mb) {
              const uint32_t ta = tmem_base + lane_addr + p.v_col0 + mb * p.n_p + 2 * g;
              float v[2];
              tmem_ld2(ta, v);
              tmem_wait_ld();
              tmem_st2(ta, v[0] * alpha, v[1] * alpha);
            }
            tmem_wait_st();
            tc_fence_before();
          }
          if (cnt < kTile && wgi == 0) {
            // rows past the context: zero them in the loaded boxes of the V stage, so
            // that the V MMA takes zero weights times zeros whatever the cache holds
            const uint32_t vs = it % p.nst_v, vph = (it / p.nst_v) & 1u;   // partial tiles only
            ok = ok && mbar_wait(&full_v[vs], vph, abort_flag);
            if (!valid) {
              const uint32_t rbytes = (uint32_t)p.cvb * 2;                 // bytes of a box row
              unsigned char* vrow = sm + p.stv_off + vs * p.stv_bytes + row * rbytes;
              for (int bx = 0; bx < p.nvb; ++bx)
                for (uint32_t c = 0; c < rbytes; c += 16)
                  *reinterpret_cast<uint4*>(vrow + bx * p.vbox_bytes + c) = make_uint4(0, 0, 0, 0);
            }
          }
          const float pj = valid ? exp2f(sc - m_ref) : 0.f;
          l_part = l_part * alpha + pj;
          const __nv_bfloat16 hi = __float2bfloat16_rn(pj);
          const __nv_bfloat16 lo = __float2bfloat16_rn(pj - __bfloat162float(hi));
          // weight rows 2g (hi) and 2g + 1 (lo): row group (2g) / 8, rows (2g) % 8 and + 1
          unsigned char* pg = sm + p.p_off + pb * p.p_buf_bytes + ((2 * g) >> 3) * 2048 +
                              (row >> 3) * 128 + ((2 * g) & 7) * 16 + (row & 7) * 2;
          *reinterpret_cast<__nv_bfloat16*>(pg) = hi;
          *reinterpret_cast<__nv_bfloat16*>(pg + 16) = lo;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pfull[pb]);   // one arrival per warp of the group
        }
        if (!ok) *abort_flag = 1;
        advance_rope(pos_next);
        pos_next = cursor_pos(p, pc, row);
        cursor_next(p, ctx_s, pc);
      }
      if (aborted) break;
      // ---------------------------------------------------------- item partial
      if (fin && r.ntiles > 0) {
        const int g = wgi;
        const size_t bh = (size_t)r.b * p.H + r.hg * HP + g;
        float* part_out = p.partials + (bh * p.S + r.s) * (2 + p.r_v);
        const float l = warp_sum_f(l_part);
        if (lane == 0) red[g * 4 + sub] = l;
        const uint32_t last = it - 1;
        const bool okv =
            __all_sync(0xffffffffu, mbar_wait(&pempty[last & 1u], (last >> 1) & 1u, abort_flag));
        tc_fence_after();
        named_barrier(2 + wgi, 128);
        if (okv) {
          if (row == 0) {
            part_out[0] = m_ref;
            part_out[1] = red[g * 4] + red[g * 4 + 1] + red[g * 4 + 2] + red[g * 4 + 3];
          }
          for (int mb = 0; mb < p.m_v; ++mb) {
            float v[2];
            tmem_ld2(tmem_base + lane_addr + p.v_col0 + mb * p.n_p + 2 * g, v);
            tmem_wait_ld();
            const int m = mb * 128 + row;            // latent dim held by this lane
            if (m < p.r_v) part_out[2 + m] = v[0] + v[1];
          }
        }
        tc_fence_before();
        named_barrier(2 + wgi, 128);
      } else if (fin) {
        const size_t bh = (size_t)r.b * p.H + r.hg * HP + wgi;
        for (int m = row; m < 2 + p.r_v; m += 128)
          p.partials[(bh * p.S + r.s) * (2 + p.r_v) + m] = m == 0 ? -INFINITY : 0.f;
        named_barrier(2 + wgi, 128);
      }
      if constexpr (FUSE) if (fin) {
        // one split per group: finalize head wgi right away.  Scratch: this
        // warpgroup's slice of the partial-exchange buffer of the parity no tile
        // touches until every warpgroup has passed the next tile's barrier.
        unsigned char* scratch = reinterpret_cast<unsigned char*>(
            sbuf + ((((it - 1u) & 1u) * HP + wgi) * kEpiWG2) * kTile);
        combine_head(p, r.b, r.hg * HP + wgi, scratch, row, 2 + wgi);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
  if (threadIdx.x == 0) {
    if (*abort_flag) atomicOr(p.status, LLA_STATUS_TIMEOUT);
    if constexpr (FUSE) {
      // the last CTA to finish publishes this call's status bits (word 1)
      __threadfence();
      if (atomicAdd(&p.counters[(size_t)p.B * p.H], 1u) == gridDim.x - 1) {
        __threadfence();
        p.status[1] = atomicExch(&p.status[0], 0);
      }
    }
  }
}

// ------------------------------------------------------------------ phase-operand kernel
//
// Per head, small latent ranks.  The score of history token j is (decode_prep_kernel's
// reordering)
//   s_j = Re sum_i U_{j,i} e^{i p_j theta_i},   U_j = c_j A~ + M~,
// with A~ = kappa conj(q~) W~ the query-absorbed up-projection and M~ its bias.
// With E_j = (cos p_j theta_i, -sin p_j theta_i)_i (two entries per RoPE pair) and
// B_m = (Re A~_{m,i}, Im A~_{m,i})_i for latent index m,
//   s_j = sum_m c_{j,m} F_{j,m} + F_{j,M},   F = E B^T,
// where F_{j,M} is the same product for the bias row M~.  E depends only on the
// tokens' positions, so one MMA per 128-token tile (M = 128, K = d, N = G r_k + 16:
// the G heads' rows B_m plus their bias rows as bf16 hi + lo) gives F for every head
// of the item, and the epilogue finishes each token-head with r_k FMAs against its
// latents instead of d/2 complex products.  The V sum is taken transposed for the G
// heads at once, D_v^T[G r_v x 2G] += C_v^T P^T, of which only the diagonal blocks
// are read (as in the LLA-2D kernel).  Both are exact reorderings of the same sums.

// Operand image of one item (sequence b, group of G heads) for decode_tcf_kernel:
// [n_f rows x d] bf16 in the 128-byte-swizzled K-major layout (d / 64 column blocks
// of n_f x 128 bytes; 16-byte chunk c of row n at chunk c ^ (n % 8)).  Row g r_k + m
// is B_m of head g, rows G r_k + 2g and + 1 its bias M~ as bf16 hi and lo, the rest
// zero.  One CTA of 128 threads per (h, b).
//
// With a phase table (table non-null) the grid also writes, from the fp32 RoPE table,
// rows [0, t_rows) of the phase table: row p holds (cos p theta_i, -sin p theta_i) as
// bf16 at entries (2i, 2i + 1), the row of E for a token at position p.  And warp w of
// CTA (h, b) marks tiles 4h + w, 4h + w + 4H, ... of sequence b: tile_p0[b][k] is the
// position of the tile's first token when every token of the tile within the context
// sits at that position plus its offset in the tile and the tile's rows lie inside
// the table, else -1; such a tile's E is rows p0 .. p0 + 127 of the table.
//
// Each CTA stages its head's W_up,k ([d][KP] fp32) and mu in shared memory with
// coalesced 16-byte reads (every CTA of a head reads the same 8-16 KB from L2), and
// every read that depends on nothing else (weights, query, q_pos, ctx_len, the first
// tile's positions, a table row) is issued before the first wait.
template <int D, int KP>
__global__ void __launch_bounds__(128) decode_prep_f_kernel(
    const float* __restrict__ q, const int32_t* __restrict__ q_pos, const float2* __restrict__ rope,
    int rope_max_pos, const float* __restrict__ wupk_t, const float* __restrict__ muk_t, float kappa,
    int H, int G, int n_f, uint32_t img_bytes, unsigned char* __restrict__ ops, int32_t* status,
    uint32_t* counters, const int32_t* __restrict__ positions, const int32_t* __restrict__ ctx_len,
    int n_cap, int n_tiles_cap, int32_t* __restrict__ tile_p0, uint32_t* __restrict__ table,
    int t_rows) {
  constexpr int HALF = D / 2;
  constexpr int EBLK = D / 64;
  constexpr int WS = KP + 1;                     // padded row of the staged weights
  constexpr int NW4 = D * KP / 4 / 128;          // 16-byte weight reads per thread
  // the partial kernel may start its prologue and latent loads now; it waits for
  // this grid before it reads the images, the table, the tile marks or the counter
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float2 qc[HALF];
  __shared__ float ws[D * WS];
  __shared__ float mus[D];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int g = h % G;
  if (counters && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0)
    counters[(size_t)gridDim.y * H] = 0u;

  // ---- reads that depend on nothing else
  const int qp_raw = q_pos[b];
  const float* qh = q + ((size_t)b * H + h) * D;
  float x0 = 0.f, x1 = 0.f;
  if (tid < HALF) {
    x0 = qh[tid];
    x1 = qh[tid + HALF];
  }
  const float4* W4 = reinterpret_cast<const float4*>(wupk_t + (size_t)h * D * KP);   // [d][KP]
  float4 w4[NW4];
#pragma unroll
  for (int j = 0; j < NW4; ++j) w4[j] = W4[tid + 128 * j];
  const float mu_v = tid < D ? muk_t[(size_t)h * D + tid] : 0.f;
  const size_t n_pairs = table ? (size_t)t_rows * HALF : 0;
  const size_t t_stride = (size_t)gridDim.x * gridDim.y * 128;
  const size_t t_idx0 = ((size_t)b * gridDim.x + h) * 128 + tid;
  float2 te = make_float2(0.f, 0.f);
  if (t_idx0 < n_pairs) te = rope[t_idx0];      // (cos, sin) of pair idx % HALF at idx / HALF
  const int k0 = 4 * h + warp;                  // this warp's first tile
  int n = 0, pv[4] = {0, 0, 0, 0};              // lane l holds offsets 4l .. 4l + 3
  auto load_tile = [&](int k) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = k * kTile + lane * 4 + e;
      pv[e] = t < n_cap ? positions[(size_t)b * n_cap + t] : 0;
    }
  };
  if (table) {
    n = ctx_len[b];
    if (k0 < n_tiles_cap) load_tile(k0);
  }
#pragma unroll
  for (int j = 0; j < NW4; ++j) {
    const int f = 4 * (tid + 128 * j), i = f / KP, m = f % KP;   // 4 | KP: one row
    float* dst = ws + i * WS + m;
    dst[0] = w4[j].x;
    dst[1] = w4[j].y;
    dst[2] = w4[j].z;
    dst[3] = w4[j].w;
  }
  if (tid < D) mus[tid] = mu_v;

  // ---- the query's RoPE factors (wait for q_pos)
  int qp = qp_raw;
  if (qp < 0 || qp >= rope_max_pos) {
    if (tid == 0 && h == 0) atomicOr(status, LLA_STATUS_POSITION_RANGE);
    qp = 0;
  }
  if (tid < HALF) {
    const float2 e = rope[(size_t)qp * HALF + tid];
    qc[tid] = make_float2(x0 * e.x - x1 * e.y, x0 * e.y + x1 * e.x);
  }

  // ---- table rows and tile marks while those land
  if (table) {
    auto put = [&](size_t idx, float2 e) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(e.x, -e.y);
      uint32_t u;
      memcpy(&u, &v, 4);
      table[idx] = u;
    };
    if (t_idx0 < n_pairs) put(t_idx0, te);
    for (size_t idx = t_idx0 + t_stride; idx < n_pairs; idx += t_stride) put(idx, rope[idx]);
    n = n < 0 ? 0 : (n > n_cap ? n_cap : n);   // the decode kernel flags a bad length
    for (int k = k0; k < n_tiles_cap; k += 4 * H) {
      if (k != k0) load_tile(k);
      const int cnt = min(kTile, n - k * kTile);
      const int p0 = __shfl_sync(0xffffffffu, pv[0], 0);
      bool ok = cnt > 0 && p0 >= 0 && p0 <= t_rows - cnt;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int off = lane * 4 + e;
        ok = ok && (off >= cnt || (uint32_t)pv[e] == (uint32_t)p0 + (uint32_t)off);
      }
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) tile_p0[(size_t)b * n_tiles_cap + k] = ok ? p0 : -1;
    }
  }
  __syncthreads();

  // ---- the image rows: this head's KP rows (W_up,k), its two bias rows (mu), and
  // (first head of the group) the zero rows that pad n_f; chunk idx is 16-byte chunk c
  // of column block kb of local row lr
  unsigned char* img = ops + ((size_t)b * (H / G) + h / G) * img_bytes;
  const int pad0 = G * KP + 2 * G;
  const int rows = KP + 2 + (g == 0 ? n_f - pad0 : 0);
  for (int idx = tid; idx < rows * EBLK * 8; idx += 128) {
    const int lr = idx / (EBLK * 8), kb = (idx >> 3) % EBLK, c = idx & 7;
    const int nr = lr < KP ? g * KP + lr
                           : (lr < KP + 2 ? G * KP + 2 * g + (lr - KP) : pad0 + (lr - KP - 2));
    __align__(16) __nv_bfloat16 v[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = kb * 32 + c * 4 + e;       // RoPE pair of entries 2e, 2e + 1
      const float2 z = qc[i];
      float re = 0.f, im = 0.f;
      if (lr < KP) {
        const float wr = ws[i * WS + lr], wi = ws[(i + HALF) * WS + lr];
        re = kappa * (z.x * wr + z.y * wi);
        im = kappa * (z.x * wi - z.y * wr);
      } else if (lr < KP + 2) {
        const float mr = mus[i], mi = mus[i + HALF];
        re = kappa * (z.x * mr + z.y * mi);
        im = kappa * (z.x * mi - z.y * mr);
        if (lr == KP + 1) {   // lo row: what the bf16 hi row leaves
          re -= __bfloat162float(__float2bfloat16_rn(re));
          im -= __bfloat162float(__float2bfloat16_rn(im));
        }
      }
      v[2 * e] = __float2bfloat16_rn(re);
      v[2 * e + 1] = __float2bfloat16_rn(im);
    }
    *reinterpret_cast<uint4*>(img + (size_t)kb * n_f * 128 + (size_t)nr * 128 + ((c ^ (nr & 7)) << 4)) =
        *reinterpret_cast<const uint4*>(v);
  }
}

// bf16 pair (low half first) -> two floats
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Warps of decode_tcf_kernel: 0 K latent producer (and each item's operand image),
// 1 F MMA issuer, 2 .. 17 epilogue (four warpgroups: warpgroup w owns head w of the
// item for scores, softmax and weights, and a quarter of the RoPE pairs of the phase
// tiles it writes), 18 V latent producer, 19 V MMA issuer.
constexpr int kGF = 4;                          // heads per item (G r_v = 128)
constexpr int kEpiWGF = 4;
constexpr int kEpiThreadsF = 128 * kEpiWGF;
constexpr int kEpiWarpsF = kEpiThreadsF / 32;
constexpr int kThreadsF = 64 + kEpiThreadsF + 64;
constexpr int kVProdWarpF = 2 + kEpiWarpsF, kVMmaWarpF = 3 + kEpiWarpsF;

// D: head width; KP: r_k (16 or 32).  r_v = 32, so the G = 4 heads' V latents fill
// the M = 128 of the transposed V MMA.
template <int D, int KP, bool FUSE>
__global__ void __launch_bounds__(kThreadsF, 1)
    decode_tcf_kernel(const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v,
                      const __grid_constant__ CUtensorMap map_e, const __grid_constant__ TcParams p) {
  constexpr int G = kGF;
  constexpr int WG_PAIRS = D / 2 / kEpiWGF;  // RoPE pairs of a token row each warpgroup writes
  constexpr uint32_t NACC = 3;               // F buffers in TMEM
  constexpr int BOXK = 64;                   // K latent boxes: 64 columns, 128-byte swizzled rows
  static_assert(WG_PAIRS % 4 == 0 && KP % 16 == 0, "shape");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full_k = reinterpret_cast<uint64_t*>(sm + p.bar_off);   // [nst] K latent tile landed
  uint64_t* empty_k = full_k + p.nst;                                // [nst] epilogue read it
  uint64_t* full_v = empty_k + p.nst;                                // [nst_v] V latent tile landed
  uint64_t* empty_v = full_v + p.nst_v;                              // [nst_v] V MMA done with it
  uint64_t* efull = empty_v + p.nst_v;   // [2] phase tile written
  uint64_t* tfull = efull + 2;           // [3] F in TMEM
  uint64_t* tempty = tfull + 3;          // [3] F read
  uint64_t* bfull = tempty + 3;          // [2] item operand image loaded
  uint64_t* bempty = bfull + 2;          // [2] operand buffer free
  uint64_t* pfull = bempty + 2;          // [2] softmax weights written
  uint64_t* pempty = pfull + 2;          // [2] V MMA done with the weights buffer
  uint64_t* drain = pempty + 2;          // [2] each MMA issuer's last MMAs completed
  uint64_t* etx = drain + 2;             // [2] phase tile's table copy landed (or none issued)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + p.misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + p.misc_off + 4);
  // how this CTA gets its phase tiles (kPhase*), written by the epilogue before its
  // first hand-off
  volatile int* phase_mode_s = reinterpret_cast<volatile int*>(sm + p.misc_off + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* ctx_s = p.B <= kCtxCache ? reinterpret_cast<const int*>(sm + p.ctx_off) : nullptr;
  // Hand-off waits (LLA_TC_POLL): 2, the default, polls with a nap between polls (the
  // epilogue LLA_TC_ENAP ns, 64; the MMA issuers LLA_TC_NAP ns, 150, in a CTA with
  // table tiles, LLA_TC_CNAP ns, 1000, in one without, known after their first
  // hand-off); 1 polls; 0 suspends.  Measured on the 21.3x workload: with every phase
  // tile computed, polling took 537-545 us per call on some B200s and 570-632 us on
  // others (same code, same clocks), napping 561-570 us on both kinds, and an MMA nap
  // of 150 ns 552 us against 540 us at 1000 ns; with table tiles the F MMA issuer also
  // waits for the tile's copy, and MMA naps of 0-300 ns took 347-351 us per call
  // against 369 us at 1000 ns, while polling everywhere took 425 us.
  uint32_t mma_nap = p.nap_ns;
  auto set_mma_nap = [&]() { mma_nap = *phase_mode_s == kPhaseComputed ? p.cnap_ns : p.nap_ns; };
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    return p.poll == 2 ? mbar_wait_nap(bar, parity, abort_flag, p.enap_ns, p.spins)
           : p.poll    ? mbar_wait_poll(bar, parity, abort_flag)
                       : mbar_wait(bar, parity, abort_flag);
  };
  auto wait_mma = [&](uint64_t* bar, uint32_t parity) {
    return p.poll == 2 ? mbar_wait_nap(bar, parity, abort_flag, mma_nap, p.spins)
           : p.poll    ? mbar_wait_poll(bar, parity, abort_flag)
                       : mbar_wait(bar, parity, abort_flag);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full_k[s], 1);
      mbar_init(&empty_k[s], kEpiWarpsF);
    }
    for (int s = 0; s < p.nst_v; ++s) {
      mbar_init(&full_v[s], 1);
      mbar_init(&empty_v[s], 1);
    }
    for (int a = 0; a < 3; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiWarpsF);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&efull[a], kEpiWarpsF);
      mbar_init(&bfull[a], 1);
      mbar_init(&bempty[a], 1);
      mbar_init(&pfull[a], kEpiWarpsF);
      mbar_init(&pempty[a], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(&etx[0], 1);
    mbar_init(&etx[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 2 + kEpiWarpsF) {
    const int et = threadIdx.x - 64;
    if (ctx_s) {
      int* cs = reinterpret_cast<int*>(sm + p.ctx_off);
      for (int b = et; b < p.B; b += kEpiThreadsF) {
        int n = p.ctx_len[b];
        if (n < 0 || n > p.n_cap) {
          if (blockIdx.x == 0) atomicOr(p.status, LLA_STATUS_CTX_RANGE);
          n = n < 0 ? 0 : p.n_cap;
        }
        cs[b] = n;
      }
    }
    if (et < 64) {
      reinterpret_cast<float2*>(sm + p.rope_off)[et] = p.step[et];
      reinterpret_cast<uint2*>(sm + p.rope_off + 512)[et] = make_uint2(p.phi_lo[et], p.phi_hi[et]);
    }
    // both weight buffers start zero: rows >= 2G are never written
    for (int idx = et; idx < 2 * 4096 / 4; idx += kEpiThreadsF)
      reinterpret_cast<uint32_t*>(sm + p.p_off)[idx] = 0u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == kVProdWarpF) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool kside = warp == 0;
      const CUtensorMap* map = kside ? &map_k : &map_v;
      tma_prefetch_desc(map);
      const int nst = kside ? p.nst : p.nst_v;
      uint64_t* fullb = kside ? full_k : full_v;
      uint64_t* emptyb = kside ? empty_k : empty_v;
      uint32_t it = 0, jn = 0;
      RingPos rs;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        if (r.ntiles == 0) continue;
        if (kside) {
          // the item's operand image (written by the prep grid, which may still be
          // running when this kernel starts)
          if (jn == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
          const uint32_t buf = jn % p.nbuf_b, bph = (jn / p.nbuf_b) & 1u;
          if (!mbar_wait(&bempty[buf], bph ^ 1u, abort_flag)) break;
          const size_t unit = (size_t)r.b * p.HG + r.hg;
          mbar_arrive_expect_tx(&bfull[buf], p.b_img_bytes);
          bulk_load(sm + p.b_off + buf * p.b_head_bytes, p.ops_b + unit * p.b_img_bytes,
                    p.b_img_bytes, &bfull[buf]);
          ++jn;
        }
        for (int k = 0; k < r.ntiles; ++k, ++it, rs.next(nst)) {
          const uint32_t stage = rs.slot, ph = rs.phase;
          if (!mbar_wait(&emptyb[stage], ph ^ 1u, abort_flag)) {   // producers suspend
            ok = false;
            break;
          }
          const int y = r.tok0 + k * kTile;
          if (kside) {
            mbar_arrive_expect_tx(&fullb[stage], p.tx_bytes);
            unsigned char* st = sm + p.st_off + stage * p.st_bytes;
            for (int kb = 0; kb < p.nkb; ++kb)
              tma_load_3d(st + kb * p.box_bytes, map, &fullb[stage],
                          r.hg * (G * KP) + kb * BOXK, y, r.b);
          } else {
            mbar_arrive_expect_tx(&fullb[stage], p.tx_v);
            unsigned char* st = sm + p.stv_off + stage * p.stv_bytes;
            for (int vb = 0; vb < p.nvb; ++vb)
              tma_load_3d(st + vb * p.vbox_bytes, map, &fullb[stage],
                          r.hg * (G * p.r_v) + vb * p.cvb, y, r.b);
          }
        }
      }
      if (*abort_flag) {
        // Drain: wait (bounded) for every copy this thread issued before leaving.
        const uint32_t n_out = it < (uint32_t)nst ? it : (uint32_t)nst;
        for (uint32_t j = 0; j < n_out; ++j) {
          const uint32_t i = it - 1 - j;
          const uint32_t stage = i % nst, ph = (i / nst) & 1u;
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&fullb[stage], ph) && global_timer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
        for (uint32_t j = 0; kside && j < (uint32_t)p.nbuf_b && j < jn; ++j) {
          const uint32_t i = jn - 1 - j;
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&bfull[i % p.nbuf_b], (i / p.nbuf_b) & 1u) &&
                 global_timer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ F MMA issuer
    // F[acc] = E (128 tokens x d, K-major) x B^T (n_f rows x d, K-major): K = d in
    // steps of 16, each a 32-byte slice of a 128-byte-swizzled column block.
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, p.n_f);
      const uint32_t e_base = smem_addr(sm + p.e_off);
      const uint32_t b_base0 = smem_addr(sm + p.b_off);
      uint32_t it = 0, jn = 0;
      RingPos ra;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        if (r.ntiles == 0) continue;
        const uint32_t buf = jn % p.nbuf_b, bph = (jn / p.nbuf_b) & 1u;
        if (!wait_mma(&bfull[buf], bph)) break;
        ++jn;
        const uint32_t b_base = b_base0 + buf * p.b_head_bytes;
        for (int k = 0; k < r.ntiles; ++k, ++it, ra.next(NACC)) {
          const uint32_t e = it & 1u, eph = (it >> 1) & 1u;     // two phase buffers
          const uint32_t acc = ra.slot, aph = ra.phase;
          if (!wait_mma(&efull[e], eph) || !wait_mma(&etx[e], eph) ||
              !wait_mma(&tempty[acc], aph ^ 1u)) {
            ok = false;
            break;
          }
          if (it == 0) set_mma_nap();
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * p.n_f;
          const uint32_t e_addr = e_base + e * p.e_bytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t blk = kk >> 2, koff = (kk & 3) * 32;
            const uint64_t adesc = smem_desc(e_addr + blk * (kTile * 128) + koff, 16, 1024, 2);
            const uint64_t bdesc = smem_desc(b_base + blk * (p.n_f * 128) + koff, 16, 1024, 2);
            mma_bf16(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&tfull[acc]);
          if (k == r.ntiles - 1) mma_commit(&bempty[buf]);   // last use of this image
        }
      }
      mma_drain(&drain[0]);
    }
    __syncwarp();
  } else if (warp == kVMmaWarpF) {
    // ------------------------------------------------------------ V MMA issuer
    // D_v^T (G r_v = 128 latent dims x 16) (+)= C_v^T (128 x 128 tokens, MN-major A,
    // two 64-dim boxes) x P^T (128 tokens x 16 weight rows, K-major B).
    if (lane == 0) {
      const uint32_t idesc_v = idesc_bf16_f32(128, 16) | (1u << 15);   // A (c_v^T) MN-major
      const uint32_t sbo_v = 16u * p.cvb;
      const uint32_t p_base = smem_addr(sm + p.p_off);
      uint32_t it = 0;
      RingPos rv;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        for (int k = 0; k < r.ntiles; ++k, ++it, rv.next(p.nst_v)) {
          const uint32_t pb = it & 1u;
          const uint32_t vs = rv.slot, vph = rv.phase;
          if (!wait_mma(&pfull[pb], (it >> 1) & 1u) || !wait_mma(&full_v[vs], vph)) {
            ok = false;
            break;
          }
          if (it == 0) set_mma_nap();
          tc_fence_after();
          const uint32_t a_addr = smem_addr(sm + p.stv_off + vs * p.stv_bytes);
          const uint32_t b_addr = p_base + pb * 4096u;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t adesc = smem_desc(a_addr + kk * 2 * sbo_v, p.vbox_bytes, sbo_v, 2);
            const uint64_t bdesc = smem_desc(b_addr + kk * 256, 128, 2048, 0);
            mma_bf16(tmem_base + p.v_col0, adesc, bdesc, idesc_v, (k == 0 && kk == 0) ? 0u : 1u);
          }
          mma_commit(&pempty[pb]);
          mma_commit(&empty_v[vs]);
        }
      }
      mma_drain(&drain[1]);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;
    const int wgi = (warp - 2) >> 2;          // warpgroup = head of the item
    const int sub = warp & 3;                 // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;          // token row of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
    float* red = reinterpret_cast<float*>(sm + p.red_off);     // [G][4]
    float* olat = reinterpret_cast<float*>(sm + p.comb_off);   // [128]: lane g r_v + m
    float* misc = olat + 128;   // [64]: m per head [0, G), q . k_self partials [8, 8 + 4G)

    // Which of this CTA's tiles take their phase rows from the table (the marks are
    // the prep grid's output).  The epilogue below is compiled three times: every
    // phase tile computed (kPhaseComputed), per tile as marked (kPhaseMixed), every
    // one copied from the table (kPhaseTable, without the RoPE factors' state).
    int phase_mode = kPhaseComputed;
    if (p.tile_p0) {
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int hit = 0, miss = 0;
      for (int item = blockIdx.x + (et >> 5) * gridDim.x; item < p.n_items;
           item += kEpiWarpsF * gridDim.x) {
        const ItemRange r = item_range(p, ctx_s, item, false);
        for (int k = lane; k < r.ntiles; k += 32) {
          const int m = __ldcg(p.tile_p0 + (size_t)r.b * p.n_tiles_cap + r.s * p.tps + k);
          hit |= m >= 0;
          miss |= m < 0;
        }
      }
      const bool any_hit = epi_barrier_or_n<kEpiThreadsF>(hit) != 0;
      const bool any_miss = epi_barrier_or_n<kEpiThreadsF>(miss) != 0;
      phase_mode = !any_hit ? kPhaseComputed : (any_miss ? kPhaseMixed : kPhaseTable);
    }
    if (et == 0) *phase_mode_s = phase_mode;   // before its first arrival on efull
    auto epilogue = [&](auto mode_tag) {
    constexpr int MODE = decltype(mode_tag)::value;
    // who needs the marks: every thread when tiles differ, the copying thread otherwise
    const bool need_mark = MODE == kPhaseMixed || (MODE == kPhaseTable && et == 0);

    // Phase tiles: the RoPE factors conj(e^{i p theta_i}) of this warpgroup's pairs at
    // this thread's token row of the last tile written, advanced by one complex
    // product when the next tile's token sits a tile further on (as in
    // decode_tc_kernel), and a cursor over the tiles still to write.  The position of
    // the next tile to write is loaded one tile before it is used, and so is its table
    // mark: a tile whose tokens sit at consecutive positions inside the phase table
    // is copied from the table's rows instead (one thread issues the copy).
    TileCursor ec;
    cursor_first(p, ctx_s, ec);
    bool e_more = ec.valid;                   // a phase tile is left to write
    // its raw position at this thread's row, and its first position in the table (or -1)
    int pos_pref = MODE == kPhaseTable ? kNoPos : cursor_pos(p, ec, row);
    int tp_pref = need_mark ? cursor_tp0(p, ec) : -1;
    int tp_cur = -1;                          // the same for the tile being written
    cursor_next(p, ctx_s, ec);
    float2 ef[WG_PAIRS];
    int pos_cur = kNoPos, run = 0;
    const float2* step_s = reinterpret_cast<const float2*>(sm + p.rope_off) + wgi * WG_PAIRS;
    const uint2* phi_s = reinterpret_cast<const uint2*>(sm + p.rope_off + 512) + wgi * WG_PAIRS;
    auto advance_rope = [&](int praw) {
      if (praw == kNoPos) return;               // row past the context: keep factors
      const int pn = checked_pos(p, praw);
      if (pos_cur != kNoPos && pn == pos_cur + kTile && run < kReseedTiles) {
#pragma unroll
        for (int q = 0; q < WG_PAIRS; ++q) {
          const float2 st = step_s[q];
          const float2 e = ef[q];
          ef[q] = make_float2(fmaf(e.x, st.x, -e.y * st.y), fmaf(e.x, st.y, e.y * st.x));
        }
        ++run;
      } else {
#pragma unroll
        for (int q = 0; q < WG_PAIRS; ++q) {
          const uint2 ph = phi_s[q];
          ef[q] = rope_factor(static_cast<uint32_t>(pn), ph.x, ph.y);
        }
        run = 0;
      }
      pos_cur = pn;
    };
#pragma unroll
    for (int q = 0; q < WG_PAIRS; ++q) ef[q] = make_float2(1.f, 0.f);
    uint32_t ie = 0;   // phase tiles written
    // The factors of the next phase tile (its position was loaded a tile ago), and the
    // position of the one after it.
    auto advance_e = [&]() {
      tp_cur = tp_pref;
      if (MODE == kPhaseComputed || (MODE == kPhaseMixed && tp_cur < 0))
        advance_rope(pos_pref);
      else
        pos_cur = kNoPos;                     // factors not kept: the next computed tile reseeds
      e_more = ec.valid;
      if (MODE != kPhaseTable) pos_pref = cursor_pos(p, ec, row);   // used by the next advance
      if (need_mark) tp_pref = cursor_tp0(p, ec);
      cursor_next(p, ctx_s, ec);
    };
    // This thread's row of that tile into buffer ie % ne: entries (2i, 2i + 1) =
    // (cos, -sin) of pair i, 128-byte swizzled K-major rows.  The caller fences and
    // arrives on efull[(ie - 1) % ne].  A table tile is one copy of D / 64 boxes of 64
    // columns x 128 rows (rows past the table read as zeros) onto etx, which the F MMA
    // issuer also waits for; a computed tile arrives on etx without a copy.
    auto store_e = [&]() {
      const uint32_t eb_i = ie & 1u;
      unsigned char* eb = sm + p.e_off + eb_i * p.e_bytes;
      if (MODE == kPhaseTable || (MODE == kPhaseMixed && tp_cur >= 0)) {
        if (et == 0) {
          mbar_arrive_expect_tx(&etx[eb_i], (uint32_t)(kTile * D * 2));
#pragma unroll
          for (int blk = 0; blk < D / 64; ++blk)
            tma_load_3d(eb + blk * (kTile * 128), &map_e, &etx[eb_i], blk * 64, tp_cur, 0);
        }
        ++ie;
        return;
      }
      if (et == 0) mbar_arrive(&etx[eb_i]);
#pragma unroll
      for (int c = 0; c < WG_PAIRS / 4; ++c) {
        const int pair0 = wgi * WG_PAIRS + c * 4;
        const int blk = pair0 >> 5, ch = (pair0 >> 2) & 7;
        uint4 v;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(ef[c * 4 + 0].x, ef[c * 4 + 0].y);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(ef[c * 4 + 1].x, ef[c * 4 + 1].y);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(ef[c * 4 + 2].x, ef[c * 4 + 2].y);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(ef[c * 4 + 3].x, ef[c * 4 + 3].y);
        memcpy(&v.x, &b0, 4);
        memcpy(&v.y, &b1, 4);
        memcpy(&v.z, &b2, 4);
        memcpy(&v.w, &b3, 4);
        *reinterpret_cast<uint4*>(eb + blk * (kTile * 128) + row * 128 + ((ch ^ (row & 7)) << 4)) = v;
      }
      ++ie;
    };
    for (int k = 0; k < 2 && e_more; ++k) {
      advance_e();
      store_e();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&efull[(ie - 1) & 1u]);
    }

    uint32_t it = 0;
    RingPos ra, rk;                           // F buffers, K stages
    bool aborted = false;
    for (int item = blockIdx.x; !aborted && item < p.n_items; item += gridDim.x) {
      const ItemRange r = item_range(p, ctx_s, item, et == 0 && !ctx_s);
      float m_ref = -INFINITY, l_part = 0.f;   // head wgi of the item
      if constexpr (FUSE) {
        // fused finish, set up while the tiles stream: the in-flight score's partial
        // dot products q . k_self (per warp), and the head's W_up,v rows into L2,
        // kept there ahead of the latent stream
        const size_t bh = (size_t)r.b * p.H + r.hg * G + wgi;
        const float qk = row < p.d ? __ldg(p.q + bh * p.d + row) * __ldg(p.k_self + bh * p.d + row) : 0.f;
        const float sdot = warp_sum_f(qk);
        if (lane == 0) misc[8 + wgi * 4 + sub] = sdot;
        const char* wrow = reinterpret_cast<const char*>(p.wupv_t + (size_t)(r.hg * G + wgi) * p.d * p.r_v);
        for (int off = row * 128; off < p.d * p.r_v * 4; off += 128 * 128)
          asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(wrow + off));
      }
      for (int k = 0; k < r.ntiles; ++k, ++it, ra.next(NACC), rk.next(p.nst)) {
        const uint32_t acc = ra.slot, aph = ra.phase;
        const uint32_t stage = rk.slot, kph = rk.phase;
        const int t0 = r.tok0 + k * kTile;
        const int cnt = min(kTile, r.tok_end - t0);
        const bool valid = row < cnt;

        bool ok = wait(&tfull[acc], aph);
        tc_fence_after();
        float f[KP];
        float fb[2];
        {
          const uint32_t col = tmem_base + lane_addr + acc * p.n_f;
#pragma unroll
          for (int c = 0; c < KP / 16; ++c) tmem_ld16(col + wgi * KP + c * 16, &f[c * 16]);
          tmem_ld2(col + G * KP + 2 * wgi, fb);
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        // the phase tile ne ahead: its factors now (arithmetic that overlaps the
        // waits below), its rows with this tile's weights
        const bool e_now = e_more;
        if (e_now) advance_e();

        // s = sum_m c_m F_m + F_M for head wgi, with this token row's latents read
        // from the swizzled K tile
        ok = ok && wait(&full_k[stage], kph);
        float sc;
        {
          const unsigned char* st = sm + p.st_off + stage * p.st_bytes;
          const int e0 = wgi * KP;                         // first latent column of the head
          const unsigned char* bx = st + (e0 / BOXK) * (kTile * BOXK * 2) + row * (BOXK * 2);
          const uint32_t c0 = (uint32_t)(e0 % BOXK) / 8;   // its first 16-byte chunk
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int cc = 0; cc < KP / 8; ++cc) {
            const uint4 w = *reinterpret_cast<const uint4*>(bx + (((c0 + cc) ^ (row & 7)) << 4));
            const float* fr = &f[cc * 8];
            a0 = fmaf(bf_lo(w.x), fr[0], a0);
            a1 = fmaf(bf_hi(w.x), fr[1], a1);
            a0 = fmaf(bf_lo(w.y), fr[2], a0);
            a1 = fmaf(bf_hi(w.y), fr[3], a1);
            a0 = fmaf(bf_lo(w.z), fr[4], a0);
            a1 = fmaf(bf_hi(w.z), fr[5], a1);
            a0 = fmaf(bf_lo(w.w), fr[6], a0);
            a1 = fmaf(bf_hi(w.w), fr[7], a1);
          }
          sc = valid ? (a0 + a1) + (fb[0] + fb[1]) : -INFINITY;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_k[stage]);
        // ---- softmax weights of head wgi against the item's reference maximum (taken
        // on the item's first tile; a later tile takes a new one only when a score
        // exceeds it by more than 2^kRescaleLog2).  One barrier of the warpgroup asks
        // whether any thread needs more than the common case: the first tile, a new
        // maximum, or a failed wait.  A warpgroup that saw a wait fail leaves the tile
        // loop; the others then find their next hand-off unanswered, time out and
        // follow, and all warpgroups agree once more before the item's finish.
        float alpha = 1.f;
        bool rescale = false;
        if (wg_barrier_or(2 + wgi, k == 0 || !ok || sc > m_ref + kRescaleLog2)) {
          if (wg_barrier_or(2 + wgi, !ok)) {
            aborted = true;
            break;
          }
          const float mx = warp_max_f(sc);
          if (lane == 0) red[wgi * 4 + sub] = mx;
          named_barrier(2 + wgi, 128);
          const float mt =
              fmaxf(fmaxf(red[wgi * 4], red[wgi * 4 + 1]), fmaxf(red[wgi * 4 + 2], red[wgi * 4 + 3]));
          if (k == 0) {
            m_ref = mt;
          } else if (mt > m_ref + kRescaleLog2) {
            alpha = exp2f(m_ref - mt);
            m_ref = mt;
            rescale = true;
          }
          named_barrier(2 + wgi, 128);   // every warp has read red before it is reused
        }
        const uint32_t pb = it & 1u;
        // the weights buffer is free once the V MMA of tile it - 2 has finished
        ok = wait(&pempty[pb], ((it >> 1) & 1u) ^ 1u);
        if (rescale) {
          // rare: rescale columns 2 wgi, 2 wgi + 1 of the V accumulator (every lane
          // this warp owns) once the V MMA of the previous tile has finished
          ok = ok && wait(&pempty[(it - 1) & 1u], ((it - 1) >> 1) & 1u);
          tc_fence_after();
          const uint32_t ta = tmem_base + lane_addr + p.v_col0 + 2 * wgi;
          float v[2];
          tmem_ld2(ta, v);
          tmem_wait_ld();
          tmem_st2(ta, v[0] * alpha, v[1] * alpha);
          tmem_wait_st();
          tc_fence_before();
        }
        if (cnt < kTile && wgi == 0) {
          // rows past the context: zero them in the V stage, so that the V MMA takes
          // zero weights times zeros whatever the cache holds there
          const uint32_t vs = it % p.nst_v, vph = (it / p.nst_v) & 1u;   // partial tiles only
          ok = ok && wait(&full_v[vs], vph);
          if (!valid) {
            unsigned char* vrow = sm + p.stv_off + vs * p.stv_bytes + row * 128;
            for (int vb = 0; vb < p.nvb; ++vb)
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(vrow + vb * p.vbox_bytes + c * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        {
          const float pj = valid ? exp2f(sc - m_ref) : 0.f;
          l_part = l_part * alpha + pj;
          const __nv_bfloat16 hi = __float2bfloat16_rn(pj);
          const __nv_bfloat16 lo = __float2bfloat16_rn(pj - __bfloat162float(hi));
          // weight rows 2 wgi (hi) and 2 wgi + 1 (lo) of row group 0
          unsigned char* pg = sm + p.p_off + pb * 4096u + (row >> 3) * 128 + ((2 * wgi) & 7) * 16 +
                              (row & 7) * 2;
          *reinterpret_cast<__nv_bfloat16*>(pg) = hi;
          *reinterpret_cast<__nv_bfloat16*>(pg + 16) = lo;
        }
        // the phase tile ne ahead goes into this tile's buffer (its last reader, this
        // tile's F MMA, has completed); one proxy fence covers both writes
        if (e_now) store_e();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pfull[pb]);               // one arrival per epilogue warp
          if (e_now) mbar_arrive(&efull[(ie - 1) & 1u]);
        }
        if (!ok) *abort_flag = 1;
      }
      if (epi_barrier_or_n<kEpiThreadsF>(aborted)) break;
      // ---------------------------------------------------------- item finish
      {
        const float l = warp_sum_f(l_part);
        if (lane == 0) red[wgi * 4 + sub] = l;
        if (row == 0) misc[wgi] = m_ref;
      }
      bool okv = true;
      if (r.ntiles > 0) {
        const uint32_t last = it - 1;
        okv = __all_sync(0xffffffffu, wait(&pempty[last & 1u], (last >> 1) & 1u));
        tc_fence_after();
      }
      named_barrier(1, kEpiThreadsF);           // red, misc visible; olat free
      // TMEM lane g r_v + m (r_v = 32: sub-partition g) holds head g's latent dim m in
      // columns 2g (hi) and 2g + 1 (lo)
      if (wgi == 0) {
        float v[2] = {0.f, 0.f};
        if (r.ntiles > 0 && okv) {
          tmem_ld2(tmem_base + lane_addr + p.v_col0 + 2 * sub, v);
          tmem_wait_ld();
        }
        olat[row] = v[0] + v[1];
      }
      tc_fence_before();
      named_barrier(1, kEpiThreadsF);           // olat complete
      if constexpr (FUSE) {
        // One split per group: o = (W_up,v o_lat a + mu_v l a + v_self b) / (l a + b),
        // a = 2^(m - M), b = 2^(s_self - M), M = max(m, s_self) (base-2 scores).
        for (int o = et; o < G * p.d; o += kEpiThreadsF) {
          const int g = o / p.d, dd = o - g * p.d;
          const int h = r.hg * G + g;
          const size_t bh = (size_t)r.b * p.H + h;
          const float m_h = r.ntiles > 0 ? misc[g] : -INFINITY;
          const float l_h = (red[g * 4] + red[g * 4 + 1]) + (red[g * 4 + 2] + red[g * 4 + 3]);
          const float s_self = p.kappa * ((misc[8 + g * 4] + misc[8 + g * 4 + 1]) +
                                          (misc[8 + g * 4 + 2] + misc[8 + g * 4 + 3]));
          const float M = fmaxf(m_h, s_self);
          const float a = r.ntiles > 0 ? exp2f(m_h - M) : 0.f, bsf = exp2f(s_self - M);
          const float inv = 1.f / (l_h * a + bsf);
          const float* Wt = p.wupv_t + (size_t)h * p.d * p.r_v + dd;
          const float* ol = olat + g * p.r_v;
          float y0 = 0.f, y1 = 0.f;
#pragma unroll
          for (int m0 = 0; m0 < 32; m0 += 16) {
            float wv[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) wv[e] = __ldg(Wt + (size_t)(m0 + e) * p.d);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              y0 = fmaf(wv[e], ol[m0 + e], y0);
              y1 = fmaf(wv[e + 1], ol[m0 + e + 1], y1);
            }
          }
          p.out[bh * p.d + dd] = ((y0 + y1) * a + __ldg(p.muv_t + (size_t)h * p.d + dd) * (l_h * a) +
                                  __ldg(p.v_self + bh * p.d + dd) * bsf) * inv;
        }
      } else {
        // split partials (m, l, sum p c_v) of the group's heads for decode_combine_kernel
        for (int idx = et; idx < G * (2 + p.r_v); idx += kEpiThreadsF) {
          const int g = idx / (2 + p.r_v), m = idx - g * (2 + p.r_v);
          const size_t bh = (size_t)r.b * p.H + r.hg * G + g;
          float v;
          if (r.ntiles == 0)
            v = m == 0 ? -INFINITY : 0.f;
          else if (m == 0)
            v = misc[g];
          else if (m == 1)
            v = (red[g * 4] + red[g * 4 + 1]) + (red[g * 4 + 2] + red[g * 4 + 3]);
          else
            v = olat[g * p.r_v + m - 2];
          p.partials[(bh * p.S + r.s) * (2 + p.r_v) + m] = v;
        }
      }
      named_barrier(1, kEpiThreadsF);           // scratch free for the next item
    }
    if (MODE != kPhaseComputed && et == 0 && (aborted || *abort_flag)) {
      // Drain: wait (bounded) for the table copies this thread issued (the last two
      // phase tiles; a computed tile's etx phase is already complete).
      for (uint32_t j = ie > 2u ? ie - 2u : 0u; j < ie; ++j) {
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait(&etx[j & 1u], (j >> 1) & 1u) &&
               global_timer_ns() - t0 < kWaitTimeoutNs) {
        }
      }
    }
    };   // epilogue
    if (phase_mode == kPhaseTable)
      epilogue(IntTag<kPhaseTable>{});
    else if (phase_mode == kPhaseMixed)
      epilogue(IntTag<kPhaseMixed>{});
    else
      epilogue(IntTag<kPhaseComputed>{});
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
  if (threadIdx.x == 0) {
    asm volatile("griddepcontrol.wait;" ::: "memory");   // prep's counter and status writes
    if (*abort_flag) atomicOr(p.status, LLA_STATUS_TIMEOUT);
    if constexpr (FUSE) {
      // the last CTA to finish publishes this call's status bits (word 1) and clears
      // word 0; otherwise the combine pass does it
      __threadfence();
      if (atomicAdd(&p.counters[(size_t)p.B * p.H], 1u) == gridDim.x - 1) {
        __threadfence();
        p.status[1] = atomicExch(&p.status[0], 0);
      }
    }
  }
}

// ------------------------------------------------------------------ host side

bool make_map(CUtensorMap* map, const void* base, int inner, int n_cap, int B, int box_inner,
              CUtensorMapSwizzle swz) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)n_cap, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * 2 * n_cap};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)kTile, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int env_int(const char* name, int dflt) {
  const char* v = std::getenv(name);
  return v && *v ? std::atoi(v) : dflt;
}

struct TcPlan {
  bool ok = false;
  bool shared = false;    // LLA-2D kernel (G heads per item share each latent tile)
  bool fform = false;     // phase-operand kernel (decode_tcf_kernel)
  int ne = 2;             // its phase-tile buffers
  int G = 1, nst = 0, nst_v = 0, nacc = 1, nbuf_b = 2, S = 0, tps = 0;
  bool nope = false;      // decoupled RoPE: score operands carry a NoPE content column
  size_t ops_bytes = 0;   // workspace for the per-(b, h) operand images
};

// Shared-memory layout for (D, G, nst); returns total bytes (plus alignment slack).
uint32_t tc_layout(TcParams& p, int D, int G, int nst, int nst_v) {
  auto al = [](uint32_t x, uint32_t a) { return (x + a - 1) / a * a; };
  p.K_pad = (p.r_k + 15) / 16 * 16;
  p.box_k = p.K_pad % 64 == 0 ? 64 : (p.K_pad % 32 == 0 ? 32 : 16);
  p.nkb = p.K_pad / p.box_k;
  p.swz = p.box_k == 64 ? 2 : (p.box_k == 32 ? 4 : 6);
  p.box_bytes = kTile * p.box_k * 2;
  p.N_v = (p.r_v + 15) / 16 * 16;
  p.cvb = p.N_v % 64 == 0 ? 64 : (p.N_v % 32 == 0 ? 32 : 16);
  p.nvb = p.N_v / p.cvb;
  p.swz_v = p.cvb == 64 ? 2 : (p.cvb == 32 ? 4 : 6);
  p.vbox_bytes = kTile * p.cvb * 2;
  p.nmb = (p.r_v + 127) / 128;
  p.cv_off = 0;
  p.tx_bytes = G * p.nkb * p.box_bytes;          // K latent stage
  p.st_bytes = al(p.tx_bytes, 1024);
  p.tx_v = G * p.nvb * p.vbox_bytes;             // V latent stage
  p.stv_bytes = al(p.tx_v, 1024);
  p.nst = nst;
  p.nst_v = nst_v;
  uint32_t o = 0;
  p.st_off = o;
  o += nst * p.st_bytes;
  p.stv_off = o;
  o += nst_v * p.stv_bytes;
  // two buffers of the query-absorbed B operand and of the bias tile (per item)
  p.b_off = o;
  p.b_head_bytes = D * p.K_pad * 2;
  p.b_sbo = (p.K_pad / 8) * 128;
  o = al(o + 2 * G * p.b_head_bytes, 1024);
  p.bias_head_bytes = D * 16 * 2;
  p.bias_off = o;
  o = al(o + 2 * G * p.bias_head_bytes, 1024);
  p.ones_off = o;
  o += 256;
  p.p_off = o;                       // softmax weights: 2 buffers x G x (8 rows x 128 tokens)
  o += 2 * G * 8 * kTile * 2;
  p.sbuf_off = o;
  o += 2 * (kEpiWG - 1) * G * kTile * 4;
  p.comb_off = o;                    // fused finish: olat [256], up-projection halves [256], misc [32]
  o += (256 + 256 + 32) * 4;
  p.red_off = o;
  o = al(o + G * 4 * 4, 16);
  p.ctx_off = o;
  o += kCtxCache * 4;
  p.rope_off = o;            // float2 step[64], then uint2 phi[64]
  o += 64 * 8 * 2;
  p.bar_off = o;
  o += (2 * nst + 2 * nst_v + 14) * 8;
  p.misc_off = o;
  o += 16;
  return o + 1024;
}

// Shared-memory layout of the LLA-2D kernel for (D, HP heads, rings, B buffers).
uint32_t tc2d_layout(TcParams& p, int D, int HP, int nst, int nst_v, int nbuf_b) {
  auto al = [](uint32_t x, uint32_t a) { return (x + a - 1) / a * a; };
  p.K_pad = (p.r_k + 15) / 16 * 16;
  p.box_k = p.K_pad % 64 == 0 ? 64 : (p.K_pad % 32 == 0 ? 32 : 16);
  p.nkb = p.K_pad / p.box_k;
  p.swz = p.box_k == 64 ? 2 : (p.box_k == 32 ? 4 : 6);
  p.box_bytes = kTile * p.box_k * 2;
  p.N_v = (p.r_v + 15) / 16 * 16;
  p.cvb = p.N_v % 64 == 0 ? 64 : (p.N_v % 32 == 0 ? 32 : 16);
  p.nvb = p.N_v / p.cvb;
  p.swz_v = p.cvb == 64 ? 2 : (p.cvb == 32 ? 4 : 6);
  p.vbox_bytes = kTile * p.cvb * 2;
  p.m_v = (p.N_v + 127) / 128;
  p.n_p = (2 * HP + 15) / 16 * 16;
  p.p_buf_bytes = (uint32_t)p.n_p * kTile * 2;
  p.tx_bytes = p.nkb * p.box_bytes;
  p.st_bytes = al(p.tx_bytes, 1024);
  p.tx_v = p.nvb * p.vbox_bytes;
  // V stages span whole 128-row blocks of the MN-major A operand; the rows past
  // r_v only feed TMEM lanes that are never read.
  p.stv_bytes = al(p.m_v * (128 / p.cvb) * p.vbox_bytes, 1024);
  p.nst = nst;
  p.nst_v = nst_v;
  p.nbuf_b = nbuf_b;
  uint32_t o = 0;
  p.st_off = o;
  o += nst * p.st_bytes;
  p.stv_off = o;
  o += nst_v * p.stv_bytes;
  p.b_off = o;
  p.b_head_bytes = D * p.K_pad * 2;
  p.b_sbo = (p.K_pad / 8) * 128;
  o = al(o + nbuf_b * HP * p.b_head_bytes, 1024);
  p.bias_head_bytes = D * 16 * 2;
  p.bias_off = o;
  o = al(o + nbuf_b * HP * p.bias_head_bytes, 1024);
  p.ones_off = o;
  o += 256;
  p.p_off = o;
  o += 2 * p.p_buf_bytes;
  p.sbuf_off = o;
  o += 2 * kEpiWG2 * HP * kTile * 4;
  p.red_off = o;
  o = al(o + HP * 4 * 4, 16);
  p.ctx_off = o;
  o += kCtxCache * 4;
  p.rope_off = o;
  o += 64 * 8 * 2;
  p.bar_off = o;
  o += (2 * nst + 2 * nst_v + 18) * 8;
  p.misc_off = o;
  o += 16;
  return o + 1024;
}

// Shared-memory layout of decode_tcf_kernel for (D, G, rings, image buffers, phase
// buffers); r_k is a multiple of 16 and G r_v = 128.
uint32_t tcf_layout(TcParams& p, int D, int G, int nst, int nst_v, int nbuf_b, int ne) {
  auto al = [](uint32_t x, uint32_t a) { return (x + a - 1) / a * a; };
  p.K_pad = p.r_k;
  const int kw = G * p.r_k;                       // K latent columns of one item
  p.box_k = kw % 64 == 0 ? 64 : 32;
  p.nkb = kw / p.box_k;
  p.swz = p.box_k == 64 ? 2 : 4;
  p.kswz_mask = p.box_k == 64 ? 7 : 3;
  p.box_bytes = kTile * p.box_k * 2;
  p.tx_bytes = p.nkb * p.box_bytes;
  p.st_bytes = al(p.tx_bytes, 1024);
  p.N_v = p.r_v;
  p.cvb = 64;                                     // V latent boxes: 64 dims, 128-byte rows
  p.nvb = G * p.r_v / 64;
  p.swz_v = 2;
  p.vbox_bytes = kTile * 64 * 2;
  p.tx_v = p.nvb * p.vbox_bytes;
  p.stv_bytes = al(p.tx_v, 1024);
  p.n_f = G * p.r_k + 16;
  p.e_bytes = kTile * D * 2;
  p.b_img_bytes = p.n_f * D * 2;
  p.b_head_bytes = al(p.b_img_bytes, 1024);       // stride of the image buffers
  p.nst = nst;
  p.nst_v = nst_v;
  p.nbuf_b = nbuf_b;
  p.ne = ne;
  uint32_t o = 0;
  p.st_off = o;
  o += nst * p.st_bytes;
  p.stv_off = o;
  o += nst_v * p.stv_bytes;
  p.e_off = o;
  o += ne * p.e_bytes;
  p.b_off = o;
  o += nbuf_b * p.b_head_bytes;
  p.p_off = o;                                    // two weight buffers, 16 rows x 128 tokens
  o += 2 * 4096;
  p.red_off = o;
  o = al(o + G * 4 * 4, 16);
  p.comb_off = o;                                 // olat [128], misc [64]
  o += (128 + 64) * 4;
  p.ctx_off = o;
  o += kCtxCache * 4;
  p.rope_off = o;
  o += 64 * 8 * 2;
  p.bar_off = o;
  o += (2 * nst + 2 * nst_v + 20) * 8;
  p.misc_off = o;
  o += 16;
  return o + 1024;
}

// Workspace of the phase-operand path, in this order: the items' operand images
// ([B][HG] of n_f x d bf16), the phase table (rows [0, n_tiles 128 + 128) of d bf16,
// 1024-byte aligned) and the tile marks ([B][n_tiles] int32).
constexpr size_t kAlignTable = 1024;
size_t tcf_images_bytes(int B, int HG, int n_f, int d) { return (size_t)B * HG * n_f * d * 2; }
size_t tcf_table_off(int B, int HG, int n_f, int d) {
  return (tcf_images_bytes(B, HG, n_f, d) + kAlignTable - 1) / kAlignTable * kAlignTable;
}
int tcf_table_rows_cap(int n_cap) { return (n_cap + kTile - 1) / kTile * kTile + kTile; }
size_t tcf_marks_off(int B, int HG, int n_f, int d, int n_cap) {
  return tcf_table_off(B, HG, n_f, d) + (size_t)tcf_table_rows_cap(n_cap) * d * 2;
}
size_t tcf_ops_bytes(int B, int HG, int n_f, int d, int n_cap) {
  return tcf_marks_off(B, HG, n_f, d, n_cap) + (size_t)B * ((n_cap + kTile - 1) / kTile) * 4;
}

// Whether the phase-operand kernel takes the shape: per head, RoPE over the whole
// head of width 64 or 128, r_k of 16 or 32, r_v = 32 (so the G = 4 heads of an item
// fill the 128 rows of the transposed V MMA) and H a multiple of 4.  LLA_TC_FORM=u
// keeps such shapes on decode_tc_kernel.
bool tcf_shape(const lla_cfg& c) {
  const char* v = std::getenv("LLA_TC_FORM");
  if (v && v[0] == 'u') return false;
  if (c.mode != LLA_MODE_PER_HEAD || has_nope(c)) return false;
  if (c.d_head != 64 && c.d_head != 128) return false;
  if (c.r_k != 16 && c.r_k != 32) return false;
  return c.r_v == 32 && c.H % kGF == 0;
}

TcPlan tc_plan(const lla_cfg& c, int B, int n_cap) {
  TcPlan pl;
  if (n_cap <= 0 || B <= 0) return pl;
  if (c.d_head != 32 && c.d_head != 64 && c.d_head != 96 && c.d_head != 128) return pl;
  // score columns per head: the rotated dims, plus 16 (the NoPE content column and
  // zero padding) with decoupled RoPE, which only the per-head kernel takes
  const bool nope = has_nope(c);
  const int D = nope ? rotary_dims(c) + 16 : c.d_head;
  const int forced_g = env_int("LLA_TC_G", 0), forced_nst = env_int("LLA_TC_NST", 0);
  const int N_v = (c.r_v + 15) / 16 * 16;
  // Largest head group G whose TMEM columns (score accumulators plus V accumulators)
  // fit in 512 and whose shared-memory ring holds at least 2 stages; two score
  // buffers when they fit.
  int best_g = 0, best_nst = 0, best_nst_v = 0, best_nacc = 1;
  if (tcf_shape(c)) {
    // phase-operand kernel: three F buffers (3 n_f + 16 TMEM columns), two phase
    // buffers, then the most latent bytes in flight with one image buffer
    // (LLA_TCF_NBUF=2 forces two)
    const int G = kGF;
    const int nbuf_f = env_int("LLA_TCF_NBUF", 0);
    for (int ne : {2}) {
      if (best_g) continue;
      for (int nbuf : {1, 2}) {
        if (best_g || (nbuf_f && nbuf != nbuf_f) || (!nbuf_f && nbuf == 2)) continue;
        TcParams p{};
        p.r_k = c.r_k;
        p.r_v = c.r_v;
        uint32_t best_bytes = 0;
        for (int nv = 8; nv >= 2; --nv)
          for (int nk = 8; nk >= 2; --nk)
            if (tcf_layout(p, c.d_head, G, nk, nv, nbuf, ne) <= kSmemLimit &&
                nk * p.st_bytes + nv * p.stv_bytes > best_bytes) {
              best_bytes = nk * p.st_bytes + nv * p.stv_bytes;
              best_nst = nk;
              best_nst_v = nv;
            }
        if (forced_nst && best_nst > forced_nst) best_nst = forced_nst;
        if (forced_nst && best_nst_v > forced_nst) best_nst_v = forced_nst;
        if (!best_bytes || best_nst < 2 || best_nst_v < 2) continue;
        best_g = G;
        best_nacc = 3;
        pl.nbuf_b = nbuf;
        pl.ne = ne;
        pl.fform = true;
      }
    }
  }
  if (c.mode == LLA_MODE_2D) {
    // HP heads per item share each latent tile: the largest HP whose operands fit,
    // double-buffered when possible; three one-head score buffers when TMEM allows.
    for (int HP : {4, 2, 1}) {
      if (c.H % HP || best_g) continue;
      if (forced_g && HP != forced_g) continue;
      const int m_v = (N_v + 127) / 128, n_p = (2 * HP + 15) / 16 * 16;
      const int nacc = 3 * D + m_v * n_p <= 512 ? 3 : (2 * D + m_v * n_p <= 512 ? 2 : 0);
      if (!nacc) continue;
      for (int nbuf : {2, 1}) {
        TcParams p{};
        p.r_k = c.r_k;
        p.r_v = c.r_v;
        int nst = 0, nst_v = 0;
        for (int nv = 6; nv >= 2 && !nst; --nv)
          for (int nk = 6; nk >= 2; --nk)
            if (tc2d_layout(p, D, HP, nk, nv, nbuf) <= kSmemLimit) {
              nst = nk;
              nst_v = nv;
              break;
            }
        if (forced_nst && nst > forced_nst) nst = forced_nst;
        if (forced_nst && nst_v > forced_nst) nst_v = forced_nst;
        if (nst < 2 || nst_v < 2) continue;
        best_g = HP;
        best_nst = nst;
        best_nst_v = nst_v;
        best_nacc = nacc;
        pl.nbuf_b = nbuf;
        pl.shared = true;
        break;
      }
    }
  }
  for (int G : {4, 2, 1}) {
    if (pl.shared || pl.fform) break;
    if (c.H % G) continue;
    if (forced_g && G != forced_g) continue;
    int nacc = 0;
    const int vcols = G * N_v;
    if (2 * G * D + vcols <= 512) nacc = 2;
    else if (G * D + vcols <= 512) nacc = 1;
    if (!nacc) continue;
    TcParams p{};
    p.r_k = c.r_k;
    p.r_v = c.r_v;
    // deepest V ring that fits (its slots are held longest), then the deepest K ring
    int nst = 0, nst_v = 0;
    for (int nv = 8; nv >= 2 && !nst; --nv)
      for (int nk = 8; nk >= 2; --nk)
        if (tc_layout(p, D, G, nk, nv) <= kSmemLimit) {
          nst = nk;
          nst_v = nv;
          break;
        }
    if (forced_nst && nst > forced_nst) nst = forced_nst;
    if (forced_nst && nst_v > forced_nst) nst_v = forced_nst;
    if (nst < 2 || nst_v < 2) continue;
    best_g = G;
    best_nst = nst;
    best_nst_v = nst_v;
    best_nacc = nacc;
    break;
  }
  if (!best_g) return pl;
  pl.G = best_g;
  pl.nst = best_nst;
  pl.nst_v = best_nst_v;
  pl.nacc = best_nacc;
  // Context splits: the split count S minimises the busiest CTA's cost over a
  // grid of one persistent CTA per SM, where items are dealt round-robin and each
  // item costs its tiles plus a fixed start/finish charge (operand hand-over, the
  // V-accumulator drain and the partial write, about 1.6 tiles of time measured on
  // the per-head 4x workload); more than one split also pays the combine pass.
  const int n_tiles = (n_cap + kTile - 1) / kTile;
  const long long units = (long long)B * (c.H / pl.G);
  const int grid = sm_count();
  constexpr double kItemCost = 1.6, kCombineCost = 0.5;   // in tiles
  // a forced split count obeys the same bounds as a planned one: the combine merges
  // at most kMaxSplits partials per head, and a split needs at least one tile
  const int forced_s = std::min(env_int("LLA_TC_SPLITS", 0), std::min(kMaxSplits, n_tiles));
  int s_max = (int)std::max<long long>(1, (4 * grid + units - 1) / units);
  s_max = std::min(std::min(s_max, kMaxSplits), n_tiles);
  double best_cost = 1e300;
  int best_s = 1;
  for (int S = forced_s > 0 ? forced_s : 1; S <= (forced_s > 0 ? forced_s : s_max); ++S) {
    const int tpi = (n_tiles + S - 1) / S;
    const int s_eff = (n_tiles + tpi - 1) / tpi;
    const long long items = units * s_eff;
    double worst = 0.0;
    if (items > grid) {
      std::vector<double> cta(grid, 0.0);
      for (long long it = 0; it < items; ++it) {
        const int sp = (int)(it % s_eff);
        cta[it % grid] += std::min(tpi, n_tiles - sp * tpi) + kItemCost;
      }
      for (double v : cta) worst = std::max(worst, v);
    } else {
      worst = tpi + kItemCost;
    }
    const double cost = worst + (s_eff > 1 ? kCombineCost : 0.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best_s = s_eff;
    }
  }
  pl.tps = (n_tiles + best_s - 1) / best_s;
  pl.S = (n_tiles + pl.tps - 1) / pl.tps;
  const size_t K_pad = (c.r_k + 15) / 16 * 16;
  pl.ops_bytes = pl.fform ? tcf_ops_bytes(B, c.H / pl.G, pl.G * c.r_k + 16, c.d_head, n_cap)
                          : (size_t)B * c.H * ((size_t)D * K_pad * 2 + (size_t)D * 32);
  pl.nope = nope;
  pl.ok = true;
  return pl;
}

bool tc_enabled() {
  const char* v = std::getenv("LLA_DECODE_PATH");
  return !(v && std::strcmp(v, "cuda_core") == 0);
}

template <int D, int G, bool SHARED, bool NOPE>
cudaError_t launch_tc_t(const CUtensorMap& mk, const CUtensorMap& mv, const TcParams& p,
                        uint32_t smem, int grid, cudaStream_t s) {
  void (*kern)(CUtensorMap, CUtensorMap, TcParams);
  if constexpr (SHARED)
    kern = p.fuse_combine ? decode_tc2d_kernel<D, G, true, NOPE> : decode_tc2d_kernel<D, G, false, NOPE>;
  else
    kern = p.fuse_combine ? decode_tc_kernel<D, G, true, NOPE> : decode_tc_kernel<D, G, false, NOPE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (SHARED || !p.fuse_combine) {
    kern<<<grid, SHARED ? kThreads2 : kThreads, smem, s>>>(mk, mv, p);
    return cudaGetLastError();
  }
  // one-split per-head plan: programmatic dependent launch after the prep kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mk, mv, p);
}

template <int D>
cudaError_t launch_tc_d(int G, bool shared, const CUtensorMap& mk, const CUtensorMap& mv,
                        const TcParams& p, uint32_t smem, int grid, cudaStream_t s) {
  switch (G * 2 + (shared ? 1 : 0)) {
    case 2: return launch_tc_t<D, 1, false, false>(mk, mv, p, smem, grid, s);
    case 4: return launch_tc_t<D, 2, false, false>(mk, mv, p, smem, grid, s);
    case 8: return launch_tc_t<D, 4, false, false>(mk, mv, p, smem, grid, s);
    case 3: return launch_tc_t<D, 1, true, false>(mk, mv, p, smem, grid, s);
    case 5: return launch_tc_t<D, 2, true, false>(mk, mv, p, smem, grid, s);
    case 9: return launch_tc_t<D, 4, true, false>(mk, mv, p, smem, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

// Decoupled RoPE: D is the rotary branch width.
template <int D>
cudaError_t launch_tc_nope(int G, bool shared, const CUtensorMap& mk, const CUtensorMap& mv,
                           const TcParams& p, uint32_t smem, int grid, cudaStream_t s) {
  switch (G * 2 + (shared ? 1 : 0)) {
    case 2: return launch_tc_t<D, 1, false, true>(mk, mv, p, smem, grid, s);
    case 4: return launch_tc_t<D, 2, false, true>(mk, mv, p, smem, grid, s);
    case 8: return launch_tc_t<D, 4, false, true>(mk, mv, p, smem, grid, s);
    case 3: return launch_tc_t<D, 1, true, true>(mk, mv, p, smem, grid, s);
    case 5: return launch_tc_t<D, 2, true, true>(mk, mv, p, smem, grid, s);
    case 9: return launch_tc_t<D, 4, true, true>(mk, mv, p, smem, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, int KP>
cudaError_t launch_tcf_t(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& me,
                         const TcParams& p, uint32_t smem, int grid, cudaStream_t s) {
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, TcParams) =
      p.fuse_combine ? decode_tcf_kernel<D, KP, true> : decode_tcf_kernel<D, KP, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch after the prep kernel: the producers wait for its
  // grid only before the first operand-image load
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreadsF);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mk, mv, me, p);
}

cudaError_t launch_tcf(int D, int KP, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& me, const TcParams& p, uint32_t smem, int grid,
                       cudaStream_t s) {
  if (D == 128 && KP == 16) return launch_tcf_t<128, 16>(mk, mv, me, p, smem, grid, s);
  if (D == 128 && KP == 32) return launch_tcf_t<128, 32>(mk, mv, me, p, smem, grid, s);
  if (D == 64 && KP == 16) return launch_tcf_t<64, 16>(mk, mv, me, p, smem, grid, s);
  if (D == 64 && KP == 32) return launch_tcf_t<64, 32>(mk, mv, me, p, smem, grid, s);
  return cudaErrorNotSupported;
}

// table / t_rows: the phase table to write and its rows (null: no table, no marks)
cudaError_t launch_prep_f(const DecodeArgs& a, const TcParams& p, int G, uint32_t* table,
                          int t_rows, cudaStream_t s) {
  dim3 grid((unsigned)a.H, (unsigned)a.B);
  unsigned char* ob = const_cast<unsigned char*>(p.ops_b);
  int32_t* marks = const_cast<int32_t*>(p.tile_p0);
#define LLA_PREP_F(DD, KK)                                                                  \
  decode_prep_f_kernel<DD, KK><<<grid, 128, 0, s>>>(                                        \
      a.q, a.q_pos, a.rope, a.rope_max_pos, a.wupk_t, a.muk_t, a.kappa, a.H, G, p.n_f,        \
      p.b_img_bytes, ob, a.status, a.counters, a.positions, a.ctx_len, a.n_cap, p.n_tiles_cap, \
      marks, table, t_rows)
  if (a.d == 128 && a.r_k == 16)
    LLA_PREP_F(128, 16);
  else if (a.d == 128 && a.r_k == 32)
    LLA_PREP_F(128, 32);
  else if (a.d == 64 && a.r_k == 16)
    LLA_PREP_F(64, 16);
  else if (a.d == 64 && a.r_k == 32)
    LLA_PREP_F(64, 32);
  else
    return cudaErrorNotSupported;
#undef LLA_PREP_F
  return cudaGetLastError();
}

cudaError_t launch_prep(const DecodeArgs& a, const TcParams& p, cudaStream_t s) {
  const int ns = a.rd < a.d ? a.rd + 16 : a.d;      // image rows per head
  const int chunks = ns * p.K_pad / 8;
  dim3 grid((unsigned)a.H, (unsigned)a.B, (unsigned)((chunks + 127) / 128));
  unsigned char* ob = const_cast<unsigned char*>(p.ops_b);
  unsigned char* obias = const_cast<unsigned char*>(p.ops_bias);
#define LLA_PREP(DD)                                                                          \
  decode_prep_kernel<DD><<<grid, 128, 0, s>>>(a.q, a.q_pos, a.rope, a.rope_max_pos, a.wupk_t, \
                                              a.muk_t, a.kappa, a.H, a.r_k, p.K_pad, ob, obias, \
                                              a.status, a.counters, a.d)
  switch (a.rd) {
    case 32: LLA_PREP(32); break;
    case 64: LLA_PREP(64); break;
    case 96: LLA_PREP(96); break;
    case 128: LLA_PREP(128); break;
    default: return cudaErrorNotSupported;
  }
#undef LLA_PREP
  return cudaGetLastError();
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

bool decode_tc_plan(const lla_cfg& c, int B, int n_cap, int* S, int* tps, size_t* ops_bytes) {
  if (!tc_enabled()) return false;
  TcPlan pl = tc_plan(c, B, n_cap);
  if (!pl.ok) return false;
  *S = pl.S;
  *tps = pl.tps;
  *ops_bytes = pl.ops_bytes;
  return true;
}

// Launch the tensor-core partial kernel; returns cudaErrorNotSupported when the
// shape is outside this path (the caller then uses the CUDA-core kernel).
cudaError_t launch_decode_tc(const lla_cfg& c, const DecodeArgs& a, cudaStream_t s) {
  if (!tc_enabled()) return cudaErrorNotSupported;
  TcPlan pl = tc_plan(c, a.B, a.n_cap);
  if (!pl.ok || pl.S != a.S) return cudaErrorNotSupported;
  TcParams p{};
  p.H = a.H;
  p.r_k = a.r_k;
  p.r_v = a.r_v;
  // At least 120 KB so that two CTAs never share an SM (each may hold all of TMEM).
  const int ns = pl.nope ? a.rd + 16 : a.d;   // score columns per head
  uint32_t smem = pl.fform    ? tcf_layout(p, a.d, pl.G, pl.nst, pl.nst_v, pl.nbuf_b, pl.ne)
                 : pl.shared ? tc2d_layout(p, ns, pl.G, pl.nst, pl.nst_v, pl.nbuf_b)
                             : tc_layout(p, ns, pl.G, pl.nst, pl.nst_v);
  if (smem < 120u * 1024u) smem = 120u * 1024u;
  p.B = a.B;
  p.n_cap = a.n_cap;
  p.S = pl.S;
  p.tps = pl.tps;
  p.HG = a.H / pl.G;
  p.n_items = a.B * p.HG * pl.S;
  p.rope_max_pos = a.rope_max_pos;
  p.nacc = pl.nacc;
  p.acc_cols = pl.fform ? p.n_f : pl.shared ? ns : pl.G * ns;
  p.v_col0 = p.nacc * p.acc_cols;
  const int v_cols = pl.fform ? 16 : pl.shared ? p.m_v * p.n_p : pl.G * p.N_v;
  int cols = 32;
  while (cols < p.v_col0 + v_cols) cols <<= 1;
  p.tmem_cols = cols;
  p.rope = a.rope;
  for (int i = 0; i < a.rd / 2; ++i) {
    const double theta = std::pow((double)a.rope_base, -2.0 * i / (double)a.rd);
    const double turns = theta / (2.0 * 3.14159265358979323846);
    const uint64_t fx = static_cast<uint64_t>(std::ldexp(turns - std::floor(turns), 64));
    p.phi_lo[i] = static_cast<uint32_t>(fx);
    p.phi_hi[i] = static_cast<uint32_t>(fx >> 32);
    const double adv = std::fmod((double)kTile * theta, 2.0 * 3.14159265358979323846);
    p.step[i] = make_float2((float)std::cos(adv), (float)-std::sin(adv));
  }
  p.ctx_len = a.ctx_len;
  p.positions = a.positions;
  p.status = a.status;
  p.partials = a.partials;
  p.q = a.q;
  p.k_self = a.k_self;
  p.v_self = a.v_self;
  p.wupv_t = a.wupv_t;
  p.muv_t = a.muv_t;
  p.out = a.out;
  p.kappa = a.kappa;
  p.d = a.d;
  p.counters = a.counters;
  if (!a.counters) return cudaErrorNotSupported;
  // Fused only when a group has one split: its combine then runs right after the
  // group's own tiles on the same CTA.  A cross-CTA merge inside this streaming
  // kernel waits on L2 round trips behind the latent traffic (measured: far slower
  // than the separate pass), so several splits keep the combine pass.
  p.fuse_combine = pl.S == 1 ? 1 : 0;
  if (!a.ops) return cudaErrorNotSupported;
  p.ops_b = a.ops;
  p.ops_bias = a.ops + (size_t)a.B * a.H * p.b_head_bytes;
  CUtensorMap mk, mv;
  const CUtensorMapSwizzle swz = p.box_k == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : p.box_k == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
  p.poll = env_int("LLA_TC_POLL", 2);
  p.nap_ns = (uint32_t)env_int("LLA_TC_NAP", 150);
  p.cnap_ns = (uint32_t)env_int("LLA_TC_CNAP", 1000);
  p.enap_ns = (uint32_t)env_int("LLA_TC_ENAP", 64);
  p.spins = (uint32_t)env_int("LLA_TC_SPIN", 0);
  p.lat_hk = (int)a.lat_head_k;
  p.lat_hv = (int)a.lat_head_v;
  if (pl.fform) {
    // K latents of an item: the G heads' r_k columns side by side (128- or 64-byte
    // rows); V latents: 64-dim boxes with 128-byte rows
    if (!make_map(&mk, a.ck, (int)a.lat_tok_k, a.n_cap, a.B, p.box_k, swz) ||
        !make_map(&mv, a.cv, (int)a.lat_tok_v, a.n_cap, a.B, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorNotSupported;
    // Phase table (LLA_TCF_TABLE=0 leaves every phase tile computed): rows up to the
    // cache's tile-rounded length plus one tile, within the RoPE table, and at least
    // one tile of them
    CUtensorMap me;
    std::memset(&me, 0, sizeof(me));
    uint32_t* table = nullptr;
    const int t_rows = std::min(a.rope_max_pos, tcf_table_rows_cap(a.n_cap));
    p.n_tiles_cap = (a.n_cap + kTile - 1) / kTile;
    p.tile_p0 = nullptr;
    if (env_int("LLA_TCF_TABLE", 1) != 0 && t_rows >= kTile) {
      const int HG = a.H / pl.G;
      table = reinterpret_cast<uint32_t*>(a.ops + tcf_table_off(a.B, HG, p.n_f, a.d));
      p.tile_p0 = reinterpret_cast<const int32_t*>(a.ops + tcf_marks_off(a.B, HG, p.n_f, a.d, a.n_cap));
      if (!make_map(&me, table, a.d, t_rows, 1, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorNotSupported;
    }
    const int sms = sm_count();
    cudaError_t pe = launch_prep_f(a, p, pl.G, table, t_rows, s);
    if (pe != cudaSuccess) return pe;
    const int grid = p.n_items < sms ? p.n_items : sms;
    cudaError_t e = launch_tcf(a.d, a.r_k, mk, mv, me, p, smem, grid, s);
    if (e == cudaSuccess && !p.fuse_combine) e = launch_combine(a, s);
    return e;
  }
  if (!make_map(&mk, a.ck, (int)a.lat_tok_k, a.n_cap, a.B, p.box_k, swz) ||
      !make_map(&mv, a.cv, (int)a.lat_tok_v, a.n_cap, a.B, p.cvb,
                p.cvb == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                : p.cvb == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                              : CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorNotSupported;
  const int sms = sm_count();
  cudaError_t pe = launch_prep(a, p, s);
  if (pe != cudaSuccess) return pe;
  const int grid = p.n_items < sms ? p.n_items : sms;
  cudaError_t e;
  if (pl.nope) {
    switch (a.rd) {
      case 32: e = launch_tc_nope<32>(pl.G, pl.shared, mk, mv, p, smem, grid, s); break;
      case 64: e = launch_tc_nope<64>(pl.G, pl.shared, mk, mv, p, smem, grid, s); break;
      default: return cudaErrorNotSupported;
    }
  } else {
    switch (a.d) {
      case 32: e = launch_tc_d<32>(pl.G, pl.shared, mk, mv, p, smem, grid, s); break;
      case 64: e = launch_tc_d<64>(pl.G, pl.shared, mk, mv, p, smem, grid, s); break;
      case 96: e = launch_tc_d<96>(pl.G, pl.shared, mk, mv, p, smem, grid, s); break;
      case 128: e = launch_tc_d<128>(pl.G, pl.shared, mk, mv, p, smem, grid, s); break;
      default: return cudaErrorNotSupported;
    }
  }
  if (e == cudaSuccess && !p.fuse_combine) e = launch_combine(a, s);
  return e;
}

}  // namespace lla
