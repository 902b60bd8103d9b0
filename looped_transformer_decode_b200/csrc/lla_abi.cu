// C ABI entry points: argument validation, exact bookkeeping, launch planning.
// Every check runs on the host before anything is enqueued.
#include <cstdio>
#include <cstdarg>
#include <cstring>
#include <cmath>
#include <string>

#include "lla_internal.cuh"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int ok() {
  g_err.clear();
  return LLA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape check shared by every entry point.  Returns LLA_OK or an error code.
int check_cfg(const lla_cfg* c) {
  if (!c) return fail(LLA_ERR_INVALID, "cfg is NULL");
  if (c->mode != LLA_MODE_PER_HEAD && c->mode != LLA_MODE_2D)
    return fail(LLA_ERR_INVALID, "mode %d is neither LLA_MODE_PER_HEAD nor LLA_MODE_2D", c->mode);
  if (c->T < 1 || c->T > 64) return fail(LLA_ERR_UNSUPPORTED, "T=%d outside [1, 64]", c->T);
  if (c->H < 1 || c->H > 128) return fail(LLA_ERR_UNSUPPORTED, "H=%d outside [1, 128]", c->H);
  if (c->d_head != 32 && c->d_head != 64 && c->d_head != 96 && c->d_head != 128)
    return fail(LLA_ERR_UNSUPPORTED, "d_head=%d not in {32, 64, 96, 128}", c->d_head);
  if (c->r_k < 8 || c->r_k > 256 || c->r_k % 8)
    return fail(LLA_ERR_UNSUPPORTED, "r_k=%d must be a multiple of 8 in [8, 256]", c->r_k);
  if (c->r_v < 8 || c->r_v > 256 || c->r_v % 8)
    return fail(LLA_ERR_UNSUPPORTED, "r_v=%d must be a multiple of 8 in [8, 256]", c->r_v);
  if (!(c->rope_base > 1.0f) || !std::isfinite(c->rope_base))
    return fail(LLA_ERR_INVALID, "rope_base=%g must be a finite value > 1", (double)c->rope_base);
  if (!(c->sm_scale >= 0.0f) || !std::isfinite(c->sm_scale))
    return fail(LLA_ERR_INVALID, "sm_scale=%g must be finite and >= 0", (double)c->sm_scale);
  if (c->d_rope != 0 && c->d_rope != c->d_head && c->d_rope != 32 && c->d_rope != 64)
    return fail(LLA_ERR_UNSUPPORTED, "d_rope=%d not in {0, 32, 64, d_head}", c->d_rope);
  if (c->d_rope > c->d_head)
    return fail(LLA_ERR_INVALID, "d_rope=%d above d_head=%d", c->d_rope, c->d_head);
  return LLA_OK;
}

int64_t gcd64(int64_t a, int64_t b) {
  while (b) {
    int64_t t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// a * b with overflow detection (non-negative operands).
bool mul_ok(int64_t a, int64_t b, int64_t* out) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > INT64_MAX / a) return false;
  *out = a * b;
  return true;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(LLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

}  // namespace

namespace lla {

PackedLayout packed_layout(const lla_cfg& c) {
  PackedLayout L{};
  const size_t T = c.T, H = c.H, d = c.d_head, rk = c.r_k, rv = c.r_v;
  L.L = c.mode == LLA_MODE_PER_HEAD ? c.H : 1;
  L.W = c.mode == LLA_MODE_PER_HEAD ? c.T * c.d_head : c.T * c.H * c.d_head;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  L.wupk = take(T * H * d * rk * 4);
  L.wupv = take(T * H * d * rv * 4);
  L.muk = take(T * H * d * 4);
  L.muv = take(T * H * d * 4);
  L.wdk = take((size_t)L.L * rk * L.W * 2);
  L.wdv = take((size_t)L.L * rv * L.W * 2);
  L.biask = take((size_t)L.L * rk * 4);
  L.biasv = take((size_t)L.L * rv * 4);
  L.wimgk = take((size_t)L.L * pad16(c.r_k) * L.W * 2);
  L.wimgv = take((size_t)L.L * pad16(c.r_v) * L.W * 2);
  L.total = o;
  return L;
}

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();   // a failed query leaves an error behind; clear it
    return 148;
  }
  return sms;
}

SplitPlan split_plan(const lla_cfg& c, int B, int n_cap) {
  SplitPlan p{};
  p.n_tiles = (n_cap + kTile - 1) / kTile;
  if (p.n_tiles == 0 || B <= 0) {
    p.splits = 0;
    p.tiles_per_split = 0;
    return p;
  }
  int S_tc = 0, tps_tc = 0;
  size_t ops = 0;
  if (decode_tc_plan(c, B, n_cap, &S_tc, &tps_tc, &ops)) {
    p.splits = S_tc;
    p.tiles_per_split = tps_tc;
    p.tensor_cores = true;
    p.ops_bytes = ops;
    return p;
  }
  // Aim for about four resident CTAs per SM.
  const long long units = (long long)B * c.H;
  long long want = (4 * sm_count() + units - 1) / units;
  if (want < 1) want = 1;
  if (want > kMaxSplits) want = kMaxSplits;
  if (want > p.n_tiles) want = p.n_tiles;
  p.tiles_per_split = (p.n_tiles + (int)want - 1) / (int)want;
  p.splits = (p.n_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
  return p;
}

int decode_check_args(const lla_cfg* cfg, const void* packed, const void* rope_table,
                      int32_t rope_max_pos, int32_t t, int32_t B, int32_t n_cap,
                      const int32_t* ctx_len, const float* q, const float* k_self,
                      const float* v_self, const int32_t* positions, const int32_t* q_pos,
                      const uint16_t* c_k, const uint16_t* c_v, const float* out) {
  int e = check_cfg(cfg);
  if (e) return e;
  if (t < 0 || t >= cfg->T) return fail(LLA_ERR_INVALID, "t=%d outside [0, T=%d)", t, cfg->T);
  if (B < 0 || n_cap < 0) return fail(LLA_ERR_INVALID, "B and n_cap must be >= 0");
  if (B > 65535) return fail(LLA_ERR_UNSUPPORTED, "B=%d above 65535", B);
  if (rope_max_pos < 1) return fail(LLA_ERR_INVALID, "rope_max_pos must be >= 1");
  if ((long long)B * n_cap > (1LL << 40)) return fail(LLA_ERR_UNSUPPORTED, "B * n_cap too large");
  if (B == 0) return ok();
  const void* ptrs[] = {packed, rope_table, ctx_len, q, k_self, v_self, q_pos, out};
  for (const void* p : ptrs) {
    if (!p) return fail(LLA_ERR_INVALID, "lla_decode_attn: NULL pointer argument");
    if (!aligned16(p)) return fail(LLA_ERR_INVALID, "lla_decode_attn: pointer not 16-byte aligned");
  }
  if (n_cap > 0) {
    const void* hist[] = {positions, c_k, c_v};
    for (const void* p : hist) {
      if (!p) return fail(LLA_ERR_INVALID, "lla_decode_attn: NULL history pointer");
      if (!aligned16(p)) return fail(LLA_ERR_INVALID, "lla_decode_attn: history pointer misaligned");
    }
  }
  if (has_nope(*cfg) && n_cap > 0 && !split_plan(*cfg, B, n_cap).tensor_cores)
    return fail(LLA_ERR_UNSUPPORTED,
                "decoupled RoPE (d_rope=%d) runs on the tensor-core path only",
                cfg->d_rope);
  return ok();
}

size_t partials_bytes(const lla_cfg& c, int B, int S) {
  return (size_t)B * c.H * S * (2 + c.r_v) * sizeof(float);
}

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

}  // namespace lla

using namespace lla;

extern "C" {

const char* lla_last_error(void) { return g_err.c_str(); }

const char* lla_version(void) { return "lla-b200 0.2 (sm_100a)"; }

int lla_ratio(const lla_cfg* cfg, int64_t* num, int64_t* den) {
  int e = check_cfg(cfg);
  if (e) return e;
  if (!num || !den) return fail(LLA_ERR_INVALID, "num/den is NULL");
  int64_t teacher = 2LL * cfg->T * cfg->H * cfg->d_head;
  int64_t lat = (int64_t)(cfg->r_k + cfg->r_v) * (cfg->mode == LLA_MODE_PER_HEAD ? cfg->H : 1);
  int64_t g = gcd64(teacher, lat);
  *num = teacher / g;
  *den = lat / g;
  return ok();
}

int lla_cache_bytes(const lla_cfg* cfg, int64_t tokens, int64_t layers, int teacher,
                    int64_t* bytes) {
  int e = check_cfg(cfg);
  if (e) return e;
  if (!bytes) return fail(LLA_ERR_INVALID, "bytes is NULL");
  if (tokens < 0 || layers < 0) return fail(LLA_ERR_INVALID, "tokens and layers must be >= 0");
  int64_t per = teacher ? 2LL * cfg->T * cfg->H * cfg->d_head
                        : (int64_t)(cfg->r_k + cfg->r_v) *
                              (cfg->mode == LLA_MODE_PER_HEAD ? cfg->H : 1);
  int64_t a, b, r;
  if (!mul_ok(per, 2, &a) || !mul_ok(a, tokens, &b) || !mul_ok(b, layers, &r))
    return fail(LLA_ERR_INVALID, "cache size overflows int64");
  *bytes = r;
  return ok();
}

size_t lla_codec_packed_bytes(const lla_cfg* cfg) {
  if (check_cfg(cfg)) return 0;
  ok();
  return packed_layout(*cfg).total;
}

int lla_codec_pack(const lla_cfg* cfg, const float* W_down_k, const float* W_down_v,
                   const float* W_up_k, const float* W_up_v, const float* mu_k,
                   const float* mu_v, void* packed, size_t packed_bytes, void* stream) {
  int e = check_cfg(cfg);
  if (e) return e;
  const void* ptrs[] = {W_down_k, W_down_v, W_up_k, W_up_v, mu_k, mu_v, packed};
  for (const void* p : ptrs) {
    if (!p) return fail(LLA_ERR_INVALID, "lla_codec_pack: NULL pointer argument");
    if (!aligned16(p)) return fail(LLA_ERR_INVALID, "lla_codec_pack: pointer not 16-byte aligned");
  }
  PackedLayout L = packed_layout(*cfg);
  if (packed_bytes < L.total)
    return fail(LLA_ERR_TOO_SMALL, "packed buffer has %zu bytes, needs %zu", packed_bytes, L.total);
  cudaError_t ce = launch_pack(*cfg, L, W_down_k, W_down_v, W_up_k, W_up_v, mu_k, mu_v,
                               static_cast<char*>(packed), static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce, "lla_codec_pack launch");
  return ok();
}

size_t lla_rope_table_bytes(const lla_cfg* cfg, int32_t max_pos) {
  if (check_cfg(cfg) || max_pos < 0) return 0;
  ok();
  return (size_t)max_pos * (rotary_dims(*cfg) / 2) * sizeof(float2);
}

int lla_rope_table(const lla_cfg* cfg, int32_t max_pos, void* table, size_t table_bytes,
                   void* stream) {
  int e = check_cfg(cfg);
  if (e) return e;
  if (max_pos < 1) return fail(LLA_ERR_INVALID, "max_pos=%d must be >= 1", max_pos);
  if (!table || !aligned16(table)) return fail(LLA_ERR_INVALID, "table NULL or misaligned");
  size_t need = lla_rope_table_bytes(cfg, max_pos);
  if (table_bytes < need)
    return fail(LLA_ERR_TOO_SMALL, "rope table has %zu bytes, needs %zu", table_bytes, need);
  cudaError_t ce = launch_rope_table(*cfg, max_pos, static_cast<float2*>(table),
                                     static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce, "lla_rope_table launch");
  return ok();
}

int lla_encode(const lla_cfg* cfg, const void* packed, int64_t n_tok, const uint16_t* x_k,
               const uint16_t* x_v, const int64_t* slot, int64_t n_slots, uint16_t* c_k,
               uint16_t* c_v, int32_t* status, void* stream) {
  int e = check_cfg(cfg);
  if (e) return e;
  if (n_tok < 0 || n_slots < 0) return fail(LLA_ERR_INVALID, "n_tok and n_slots must be >= 0");
  if (n_tok == 0) return ok();
  if (n_tok > (int64_t)INT32_MAX) return fail(LLA_ERR_UNSUPPORTED, "n_tok above 2^31-1");
  const void* ptrs[] = {packed, x_k, x_v, slot, c_k, c_v};
  for (const void* p : ptrs) {
    if (!p) return fail(LLA_ERR_INVALID, "lla_encode: NULL pointer argument");
    if (!aligned16(p)) return fail(LLA_ERR_INVALID, "lla_encode: pointer not 16-byte aligned");
  }
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u))
    return fail(LLA_ERR_INVALID, "lla_encode: status not 4-byte aligned");
  PackedLayout L = packed_layout(*cfg);
  if (L.W > 49152)
    return fail(LLA_ERR_UNSUPPORTED, "encode input width %d above 49152", L.W);
  const char* pk = static_cast<const char*>(packed);
  const auto* xk = reinterpret_cast<const __nv_bfloat16*>(x_k);
  const auto* xv = reinterpret_cast<const __nv_bfloat16*>(x_v);
  auto* ck = reinterpret_cast<__nv_bfloat16*>(c_k);
  auto* cv = reinterpret_cast<__nv_bfloat16*>(c_v);
  auto* st = static_cast<cudaStream_t>(stream);
  cudaError_t ce = launch_encode_tc(*cfg, L, pk, n_tok, xk, xv, slot, n_slots, ck, cv, status, st);
  if (ce == cudaErrorNotSupported)
    ce = launch_encode(*cfg, L, pk, n_tok, xk, xv, slot, n_slots, ck, cv, status, st);
  if (ce != cudaSuccess) return cuda_fail(ce, "lla_encode launch");
  return ok();
}

size_t lla_decode_workspace_bytes(const lla_cfg* cfg, int32_t B, int32_t n_cap) {
  if (check_cfg(cfg) || B < 0 || n_cap < 0) return 0;
  ok();
  SplitPlan p = split_plan(*cfg, B, n_cap);
  return kWsHeader + align_up(partials_bytes(*cfg, B, p.splits), 256) + align_up(p.ops_bytes, 256) +
         (p.tensor_cores ? align_up(((size_t)B * cfg->H + 1) * 4, 256) : 0);
}

int lla_decode_launches(const lla_cfg* cfg, int32_t B, int32_t n_cap) {
  if (check_cfg(cfg) || B < 0 || n_cap < 0) return -1;
  if (B == 0) return 0;
  if (n_cap == 0) return 1;
  // tensor cores: prep + partials + combine, the combine fused into the partials
  // when each per-head group has a single split; CUDA cores: partials + combine
  const SplitPlan sp = split_plan(*cfg, B, n_cap);
  if (!sp.tensor_cores) return 2;
  return sp.splits == 1 ? 2 : 3;
}

int lla_decode_attn(const lla_cfg* cfg, const void* packed, const void* rope_table,
                    int32_t rope_max_pos, int32_t t, int32_t B, int32_t n_cap,
                    const int32_t* ctx_len, const float* q, const float* k_self,
                    const float* v_self, const int32_t* positions, const int32_t* q_pos,
                    const uint16_t* c_k, const uint16_t* c_v, float* out, void* ws,
                    size_t ws_bytes, void* stream) {
  int e = lla::decode_check_args(cfg, packed, rope_table, rope_max_pos, t, B, n_cap, ctx_len, q,
                                 k_self, v_self, positions, q_pos, c_k, c_v, out);
  if (e) return e;
  if (B == 0) return ok();
  if (!ws) return fail(LLA_ERR_INVALID, "lla_decode_attn: NULL pointer argument");
  if (!aligned16(ws)) return fail(LLA_ERR_INVALID, "lla_decode_attn: pointer not 16-byte aligned");
  SplitPlan plan = split_plan(*cfg, B, n_cap);
  const size_t ops_at = kWsHeader + align_up(partials_bytes(*cfg, B, plan.splits), 256);
  const size_t counters_at = ops_at + align_up(plan.ops_bytes, 256);
  size_t need = counters_at + (plan.tensor_cores ? align_up(((size_t)B * cfg->H + 1) * 4, 256) : 0);
  if (ws_bytes < need)
    return fail(LLA_ERR_TOO_SMALL, "workspace has %zu bytes, needs %zu", ws_bytes, need);

  PackedLayout L = packed_layout(*cfg);
  const char* pk = static_cast<const char*>(packed);
  const size_t d = cfg->d_head, H = cfg->H;
  DecodeArgs a{};
  a.T = cfg->T;
  a.H = cfg->H;
  a.d = cfg->d_head;
  a.rd = rotary_dims(*cfg);
  a.r_k = cfg->r_k;
  a.r_v = cfg->r_v;
  a.mode = cfg->mode;
  float scale = cfg->sm_scale > 0.f ? cfg->sm_scale : 1.0f / std::sqrt((float)cfg->d_head);
  a.kappa = (float)((double)scale * 1.4426950408889634);  // log2(e)
  a.t = t;
  a.B = B;
  a.n_cap = n_cap;
  a.rope_max_pos = rope_max_pos;
  a.rope_base = cfg->rope_base;
  a.wupk_t = reinterpret_cast<const float*>(pk + L.wupk) + (size_t)t * H * d * cfg->r_k;
  a.wupv_t = reinterpret_cast<const float*>(pk + L.wupv) + (size_t)t * H * d * cfg->r_v;
  a.muk_t = reinterpret_cast<const float*>(pk + L.muk) + (size_t)t * H * d;
  a.muv_t = reinterpret_cast<const float*>(pk + L.muv) + (size_t)t * H * d;
  a.rope = static_cast<const float2*>(rope_table);
  a.ctx_len = ctx_len;
  a.q = q;
  a.k_self = k_self;
  a.v_self = v_self;
  a.positions = positions;
  a.q_pos = q_pos;
  a.ck = reinterpret_cast<const __nv_bfloat16*>(c_k);
  a.cv = reinterpret_cast<const __nv_bfloat16*>(c_v);
  if (cfg->mode == LLA_MODE_PER_HEAD) {
    a.lat_tok_k = (long long)H * cfg->r_k;
    a.lat_tok_v = (long long)H * cfg->r_v;
    a.lat_head_k = cfg->r_k;
    a.lat_head_v = cfg->r_v;
  } else {
    a.lat_tok_k = cfg->r_k;
    a.lat_tok_v = cfg->r_v;
    a.lat_head_k = 0;
    a.lat_head_v = 0;
  }
  a.out = out;
  a.status = static_cast<int32_t*>(ws);
  a.partials = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsHeader);
  a.S = plan.splits;
  a.tiles_per_split = plan.tiles_per_split;
  a.ops = plan.tensor_cores ? static_cast<unsigned char*>(ws) + ops_at : nullptr;
  a.counters = plan.tensor_cores
                   ? reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + counters_at)
                   : nullptr;
  int launches = 0;
  cudaError_t ce = cudaErrorNotSupported;
  if (plan.tensor_cores && plan.splits > 0)
    ce = launch_decode_tc(*cfg, a, static_cast<cudaStream_t>(stream));
  if (ce == cudaErrorNotSupported && has_nope(*cfg) && n_cap > 0)
    return fail(LLA_ERR_UNSUPPORTED, "decoupled RoPE shape not taken by the tensor-core path");
  if (ce == cudaErrorNotSupported) ce = launch_decode(a, static_cast<cudaStream_t>(stream), &launches);
  if (ce != cudaSuccess) return cuda_fail(ce, "lla_decode_attn launch");
  return ok();
}


int64_t lla_evict_slot(int32_t sink, int32_t window, int64_t pos) {
  return lla::evict_slot(sink, window, pos);
}

int lla_evict_append(int32_t B, int32_t n_cap, int32_t sink, int32_t window, const int32_t* pos,
                     int64_t* slot, int32_t* positions, int32_t* ctx_len, void* stream) {
  if (B < 0 || n_cap < 1) return fail(LLA_ERR_INVALID, "lla_evict_append: B must be >= 0 and n_cap >= 1");
  if (sink < 0 || window < 1) return fail(LLA_ERR_INVALID, "lla_evict_append: need sink >= 0 and window >= 1");
  if ((int64_t)sink + window > n_cap)
    return fail(LLA_ERR_INVALID, "lla_evict_append: sink + window = %lld exceeds n_cap = %d",
                (long long)sink + window, n_cap);
  if (B == 0) return ok();
  if (!pos || !slot || !positions || !ctx_len)
    return fail(LLA_ERR_INVALID, "lla_evict_append: NULL pointer argument");
  if ((reinterpret_cast<uintptr_t>(slot) & 7u) || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
      (reinterpret_cast<uintptr_t>(positions) & 3u) || (reinterpret_cast<uintptr_t>(ctx_len) & 3u))
    return fail(LLA_ERR_INVALID, "lla_evict_append: misaligned pointer");
  cudaError_t ce = lla::launch_evict_append(B, n_cap, sink, window, pos, slot, positions, ctx_len,
                                            static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce, "lla_evict_append launch");
  return ok();
}

// ---------------------------------------------------------------- full-memory fast path

size_t lla_full_kv_bytes(const lla_cfg* cfg, int32_t B, int32_t n_cap) {
  if (check_cfg(cfg) || B < 0 || n_cap < 0) return 0;
  return (size_t)B * cfg->H * (size_t)n_cap * cfg->d_head * 2;
}

int lla_full_rebuild(const lla_cfg* cfg, const void* packed, const void* rope_table,
                     int32_t rope_max_pos, int32_t t, int32_t B, int32_t n_cap,
                     const int32_t* positions, const uint16_t* c_k, const uint16_t* c_v,
                     const int64_t* slot, int64_t n_rows, uint16_t* k_full, uint16_t* v_full,
                     int32_t* status, void* stream) {
  int e = check_cfg(cfg);
  if (e) return e;
  if (has_nope(*cfg)) return fail(LLA_ERR_UNSUPPORTED, "the full-memory path rotates whole heads");
  if (t < 0 || t >= cfg->T) return fail(LLA_ERR_INVALID, "t=%d outside [0, T=%d)", t, cfg->T);
  if (B < 0 || n_cap < 0 || n_rows < 0)
    return fail(LLA_ERR_INVALID, "B, n_cap and n_rows must be >= 0");
  if (rope_max_pos < 1) return fail(LLA_ERR_INVALID, "rope_max_pos must be >= 1");
  if (!slot && n_rows > (int64_t)B * n_cap)
    return fail(LLA_ERR_INVALID, "n_rows=%lld above B * n_cap without a slot list",
                (long long)n_rows);
  if (n_rows == 0) return ok();
  const void* ptrs[] = {packed, rope_table, positions, c_k, c_v, k_full, v_full};
  for (const void* p : ptrs) {
    if (!p) return fail(LLA_ERR_INVALID, "lla_full_rebuild: NULL pointer argument");
    if (!aligned16(p)) return fail(LLA_ERR_INVALID, "lla_full_rebuild: pointer not 16-byte aligned");
  }
  if (slot && !aligned16(slot)) return fail(LLA_ERR_INVALID, "lla_full_rebuild: slot misaligned");
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u))
    return fail(LLA_ERR_INVALID, "lla_full_rebuild: status not 4-byte aligned");
  PackedLayout L = packed_layout(*cfg);
  const char* pk = static_cast<const char*>(packed);
  const size_t d = cfg->d_head, H = cfg->H;
  FullRebuildArgs a{};
  a.d = cfg->d_head;
  a.H = cfg->H;
  a.r_k = cfg->r_k;
  a.r_v = cfg->r_v;
  a.B = B;
  a.n_cap = n_cap;
  a.rope_max_pos = rope_max_pos;
  a.n_rows = n_rows;
  a.slot = slot;
  a.positions = positions;
  a.rope = static_cast<const float2*>(rope_table);
  a.wupk_t = reinterpret_cast<const float*>(pk + L.wupk) + (size_t)t * H * d * cfg->r_k;
  a.wupv_t = reinterpret_cast<const float*>(pk + L.wupv) + (size_t)t * H * d * cfg->r_v;
  a.muk_t = reinterpret_cast<const float*>(pk + L.muk) + (size_t)t * H * d;
  a.muv_t = reinterpret_cast<const float*>(pk + L.muv) + (size_t)t * H * d;
  a.ck = reinterpret_cast<const __nv_bfloat16*>(c_k);
  a.cv = reinterpret_cast<const __nv_bfloat16*>(c_v);
  const bool per_head = cfg->mode == LLA_MODE_PER_HEAD;
  a.lat_tok_k = per_head ? (long long)H * cfg->r_k : cfg->r_k;
  a.lat_tok_v = per_head ? (long long)H * cfg->r_v : cfg->r_v;
  a.lat_head_k = per_head ? cfg->r_k : 0;
  a.lat_head_v = per_head ? cfg->r_v : 0;
  a.k_full = reinterpret_cast<__nv_bfloat16*>(k_full);
  a.v_full = reinterpret_cast<__nv_bfloat16*>(v_full);
  a.status = status;
  cudaError_t ce = launch_full_rebuild(a, static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce, "lla_full_rebuild launch");
  return ok();
}

size_t lla_full_decode_workspace_bytes(const lla_cfg* cfg, int32_t B, int32_t n_cap) {
  if (check_cfg(cfg) || B < 0 || n_cap < 0) return 0;
  FullPlan pl = full_plan(*cfg, B, n_cap);
  const size_t parts = pl.S > 1 ? (size_t)B * cfg->H * pl.S * (cfg->d_head + 2) * 4 : 0;
  return kWsHeader + align_up(parts, 256);
}

int lla_full_decode_launches(const lla_cfg* cfg, int32_t B, int32_t n_cap) {
  if (check_cfg(cfg) || B < 0 || n_cap < 0) return -1;
  if (B == 0) return 0;
  return full_plan(*cfg, B, n_cap).S > 1 ? 2 : 1;
}

int lla_full_decode_attn(const lla_cfg* cfg, const void* rope_table, int32_t rope_max_pos,
                         int32_t B, int32_t n_cap, const int32_t* ctx_len, const float* q,
                         const float* k_self, const float* v_self, const int32_t* q_pos,
                         const uint16_t* k_full, const uint16_t* v_full, float* out, void* ws,
                         size_t ws_bytes, void* stream) {
  int e = check_cfg(cfg);
  if (e) return e;
  if (has_nope(*cfg)) return fail(LLA_ERR_UNSUPPORTED, "the full-memory path rotates whole heads");
  if (B < 0 || n_cap < 0) return fail(LLA_ERR_INVALID, "B and n_cap must be >= 0");
  if (rope_max_pos < 1) return fail(LLA_ERR_INVALID, "rope_max_pos must be >= 1");
  if ((long long)B * cfg->H * (long long)n_cap > (long long)INT32_MAX)
    return fail(LLA_ERR_UNSUPPORTED, "B * H * n_cap above 2^31-1 cache rows");
  if (B == 0) return ok();
  const void* ptrs[] = {rope_table, ctx_len, q, k_self, v_self, q_pos, out, ws};
  for (const void* p : ptrs) {
    if (!p) return fail(LLA_ERR_INVALID, "lla_full_decode_attn: NULL pointer argument");
    if (!aligned16(p))
      return fail(LLA_ERR_INVALID, "lla_full_decode_attn: pointer not 16-byte aligned");
  }
  if (n_cap > 0) {
    const void* hist[] = {k_full, v_full};
    for (const void* p : hist) {
      if (!p) return fail(LLA_ERR_INVALID, "lla_full_decode_attn: NULL cache pointer");
      if (!aligned16(p)) return fail(LLA_ERR_INVALID, "lla_full_decode_attn: cache misaligned");
    }
  }
  const size_t need = lla_full_decode_workspace_bytes(cfg, B, n_cap);
  if (ws_bytes < need)
    return fail(LLA_ERR_TOO_SMALL, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  FullPlan pl = full_plan(*cfg, B, n_cap);
  FullDecodeParams p{};
  p.B = B;
  p.H = cfg->H;
  p.n_cap = n_cap;
  p.d = cfg->d_head;
  p.S = pl.S;
  p.tps = pl.tps;
  p.n_items = (int)pl.n_items;
  p.rope_max_pos = rope_max_pos;
  p.fuse = pl.S == 1 ? 1 : 0;
  const float scale = cfg->sm_scale > 0.f ? cfg->sm_scale : 1.0f / std::sqrt((float)cfg->d_head);
  p.kappa = (float)((double)scale * 1.4426950408889634);  // log2(e): base-2 scores
  p.q = q;
  p.k_self = k_self;
  p.v_self = v_self;
  p.q_pos = q_pos;
  p.ctx_len = ctx_len;
  p.rope = static_cast<const float2*>(rope_table);
  p.out = out;
  p.status = static_cast<int32_t*>(ws);
  p.counter = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 16);
  p.partials = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsHeader);
  // with no history the tensor maps are never read; any aligned address encodes them
  const void* kb = n_cap > 0 ? static_cast<const void*>(k_full) : ws;
  const void* vb = n_cap > 0 ? static_cast<const void*>(v_full) : ws;
  cudaError_t ce = launch_full_decode(p, kb, vb, pl.grid, static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return cuda_fail(ce, "lla_full_decode_attn launch");
  return ok();
}

}  // extern "C"
