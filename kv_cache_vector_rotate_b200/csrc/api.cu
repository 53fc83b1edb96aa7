// C ABI of libtq: argument checks, codebook construction / upload, dispatch.
// The method follows "TurboQuant explained" (a2a-mcp.org), §Stage 1 and
// §Stage 2; the entry points are documented in include/tq.h.

#include <cmath>
#include <cstring>
#include <new>
#include <string>

#include "codebook_host.h"
#include "tq_internal.cuh"

namespace tq {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

tq_status fail(tq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

tq_status cuda_fail(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return TQ_OK;
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return TQ_ECUDA;
}

tq_status launch_quantize_simt(const tq_codebook* cb, const void* x, tq_dtype dt, int64_t batch,
                               int n_kv_heads, int64_t n_new, const int32_t* start_pos,
                               const CacheView& cv, cudaStream_t st);
tq_status launch_quantize_small(const tq_codebook* cb, const void* x, tq_dtype dt, int64_t batch,
                                int n_kv_heads, int64_t n_new, const int32_t* start_pos,
                                const CacheView& cv, cudaStream_t st, bool* handled);
tq_status launch_quantize_small_kv(const tq_codebook* kcb, const void* k, const tq_codebook* vcb, const void* v,
                                   tq_dtype dt, int64_t batch, int n_kv_heads, int64_t n_new,
                                   const int32_t* start_pos, const CacheView& kcv, const CacheView& vcv,
                                   cudaStream_t st, bool* handled);
tq_status launch_quantize_tc(const tq_codebook* cb, const void* x, tq_dtype dt, int64_t batch,
                             int n_kv_heads, int64_t n_new, const int32_t* start_pos,
                             const CacheView& cv, cudaStream_t st, bool* handled);

// IEEE binary16 bits of x, rounded to nearest-even directly from double.
static uint16_t f64_to_f16_bits(double x) {
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double a = std::fabs(x);
  if (a >= 65520.0) return sign | 0x7C00;
  if (a == 0.0) return sign;
  int e;
  std::frexp(a, &e);                           // a = f 2^e, f in [0.5, 1)
  const int E = std::max(e - 1, -14);          // exponent of the fp16 quantum
  const double quantum = std::ldexp(1.0, E - 10);
  const double v = std::nearbyint(a / quantum) * quantum;   // round half to even
  if (v < std::ldexp(1.0, -14)) return sign | (uint16_t)(v / std::ldexp(1.0, -24));
  std::frexp(v, &e);
  const int ev = e - 1;
  if (ev > 15) return sign | 0x7C00;
  const uint16_t mant = (uint16_t)((v / std::ldexp(1.0, ev) - 1.0) * 1024.0);
  return sign | (uint16_t)((ev + 15) << 10) | mant;
}

static float f16_bits_to_float(uint16_t h) {
  __half_raw r;
  r.x = h;
  return __half2float(__half(r));
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static tq_status check_params(const tq_params* p) {
  if (!p) return fail(TQ_EINVAL, "params is NULL");
  if (p->d < 8 || p->d > 256 || p->d % 8 != 0)
    return fail(TQ_EINVAL, "d must be a multiple of 8 in [8, 256]");
  if (p->bits < 1 || p->bits > 4) return fail(TQ_EUNSUPPORTED, "bits must be in [1, 4]");
  if (p->m < 0) return fail(TQ_EINVAL, "m must be >= 0");
  if (p->m > 0 && 64 * ((p->m + 63) / 64) != 64 * ((p->d + 63) / 64))
    return fail(TQ_EUNSUPPORTED, "m must be 0 or round up to the same multiple of 64 as d");
  return TQ_OK;
}

static void build_host_tables(tq_codebook* cb, const tq_params* p) {
  const int d = p->d, m = p->m;
  std::vector<double> G((size_t)d * d);
  tqhost::gaussian_fill(p->seed_pi, G.size(), G.data());
  cb->pi = tqhost::orthogonal_factor(G, d);
  cb->s.assign((size_t)m * d, 0.0);
  if (m > 0) tqhost::gaussian_fill(p->seed_s, cb->s.size(), cb->s.data());
  tqhost::LloydMax lm = tqhost::lloyd_max(d, p->bits);
  cb->centroids = lm.centroids;
  cb->boundaries = lm.boundaries;
  cb->s_row_norm_max = 0.0;
  for (int i = 0; i < m; ++i) {
    double s2 = 0.0;
    for (int k = 0; k < d; ++k) s2 += cb->s[(size_t)i * d + k] * cb->s[(size_t)i * d + k];
    cb->s_row_norm_max = std::max(cb->s_row_norm_max, std::sqrt(s2));
  }
  cb->qjl_scale = m > 0 ? std::sqrt(3.14159265358979323846 / 2.0) / m : 0.0;
  const int K = 1 << p->bits, H = K / 2;
  for (int i = 0; i < 16; ++i) cb->cent16[i] = 0;
  for (int i = 0; i < 8; ++i) cb->mag16[i] = 0;
  cb->table_exp = 0;
  cb->int8_levels[0] = cb->int8_levels[1] = 0u;
  cb->levels.assign(K, 0.0);
  // Reconstruction levels (TQ §Stage 1 gives the centroids, not how they are
  // stored): up to 8 levels in 8-bit fixed point on one power-of-two scale,
  // level i = k_i 2^-f with k_i = round(c_i 2^f) (half to even) and f the
  // largest integer with max |c| 2^f <= 127, so that a decoded coordinate is
  // one signed byte; 16 levels in fp16.
  if (K <= 8) {
    double cmax = 0.0;
    for (int i = 0; i < K; ++i) cmax = std::max(cmax, std::fabs(cb->centroids[i]));
    const int f = (int)std::floor(std::log2(127.0 / cmax));
    for (int i = 0; i < K; ++i) {
      const double k = std::nearbyint(std::ldexp(cb->centroids[i], f));
      cb->levels[i] = std::ldexp(k, -f);
      cb->int8_levels[i / 4] |= (uint32_t)(uint8_t)(int8_t)k << (8 * (i % 4));
    }
    cb->table_exp = f;
  } else {
    for (int i = 0; i < K; ++i) cb->levels[i] = f16_bits_to_float(f64_to_f16_bits(cb->centroids[i]));
  }
  for (int i = 0; i < K; ++i) cb->cent16[i] = f64_to_f16_bits(cb->levels[i]);   // exact
  for (int mu = 0; mu < H; ++mu) cb->mag16[mu] = cb->cent16[H + mu];
}

static tq_status upload(tq_codebook* cb) {
  const Layout& L = cb->lay;
  const int d = L.d, dp = L.d_pad, mp = L.m_pad, K = 1 << L.bits;
  auto al = [](size_t n) { return (n + 255) / 256 * 256; };
  const size_t sz_pi = al((size_t)dp * d * 4), sz_s = al((size_t)mp * d * 4 + 4),
               sz_srott = al((size_t)dp * mp * 4 + 4), sz_b = al(16 * 4), sz_c = al(16 * 4),
               sz_pibf = al((size_t)2 * dp * dp * 2), sz_srbf = al((size_t)2 * mp * dp * 2 + 4);
  const size_t sz_pit = al((size_t)d * dp * 4), sz_st = al((size_t)d * mp * 4 + 4),
               sz_srot = al((size_t)mp * dp * 4 + 4);
  const int R = dp + mp, d16 = (d + 15) / 16;
  const size_t sz_qf = al((size_t)(R / 16) * d16 * 2 * 32 * 16);
  const size_t total =
      sz_pi + sz_s + sz_srott + sz_b + sz_c + sz_pibf + sz_srbf + sz_pit + sz_st + sz_qf + sz_srot;
  std::vector<uint8_t> host(total, 0);
  size_t off = 0;
  auto take = [&](size_t n) { size_t o = off; off += n; return o; };
  const size_t o_pi = take(sz_pi), o_s = take(sz_s), o_srott = take(sz_srott), o_b = take(sz_b),
               o_c = take(sz_c), o_pibf = take(sz_pibf), o_srbf = take(sz_srbf),
               o_pit = take(sz_pit), o_st = take(sz_st), o_qf = take(sz_qf), o_srot = take(sz_srot);
  float* pi32 = reinterpret_cast<float*>(host.data() + o_pi);
  float* s32 = reinterpret_cast<float*>(host.data() + o_s);
  float* srott32 = reinterpret_cast<float*>(host.data() + o_srott);
  float* b32 = reinterpret_cast<float*>(host.data() + o_b);
  float* c32 = reinterpret_cast<float*>(host.data() + o_c);
  __nv_bfloat16* pibf = reinterpret_cast<__nv_bfloat16*>(host.data() + o_pibf);
  __nv_bfloat16* srbf = reinterpret_cast<__nv_bfloat16*>(host.data() + o_srbf);
  float* pit32 = reinterpret_cast<float*>(host.data() + o_pit);
  float* st32 = reinterpret_cast<float*>(host.data() + o_st);
  float* srot32 = reinterpret_cast<float*>(host.data() + o_srot);
  for (int j = 0; j < d; ++j)
    for (int k = 0; k < d; ++k) {
      pi32[(size_t)j * d + k] = (float)cb->pi[(size_t)j * d + k];
      pit32[(size_t)k * dp + j] = (float)cb->pi[(size_t)j * d + k];
    }
  for (int i = 0; i < L.m; ++i)
    for (int k = 0; k < d; ++k) st32[(size_t)k * mp + i] = (float)cb->s[(size_t)i * d + k];
  for (int i = 0; i < L.m; ++i)
    for (int k = 0; k < d; ++k) s32[(size_t)i * d + k] = (float)cb->s[(size_t)i * d + k];
  // S_rot = S Pi^T: the residual is formed in the rotated space, and
  // S r = S Pi^T (Pi r).
  for (int i = 0; i < L.m; ++i)
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += cb->s[(size_t)i * d + k] * cb->pi[(size_t)j * d + k];
      srott32[(size_t)j * mp + i] = (float)acc;
      srot32[(size_t)i * dp + j] = (float)acc;
      const __nv_bfloat16 hi = __double2bfloat16(acc);
      srbf[(size_t)i * dp + j] = hi;
      srbf[(size_t)mp * dp + (size_t)i * dp + j] = __double2bfloat16(acc - (double)__bfloat162float(hi));
    }
  for (int j = 0; j < d; ++j)
    for (int k = 0; k < d; ++k) {
      const double v = cb->pi[(size_t)j * d + k];
      const __nv_bfloat16 hi = __double2bfloat16(v);
      pibf[(size_t)j * dp + k] = hi;
      pibf[(size_t)dp * dp + (size_t)j * dp + k] = __double2bfloat16(v - (double)__bfloat162float(hi));
    }
  for (int i = 0; i < K - 1; ++i) b32[i] = (float)cb->boundaries[i];
  for (int i = 0; i < K; ++i) c32[i] = f16_bits_to_float(cb->cent16[i]);
  // [Pi ; S] as bf16 hi + lo A fragments of mma.m16n8k16 (row-major A): lane
  // (g, t) holds {A[g][2t], A[g][2t+1]}, {A[g+8][2t], ..}, {A[g][2t+8], ..},
  // {A[g+8][2t+8], ..} of each 16 x 16 block, low half first.
  {
    uint32_t* qf = reinterpret_cast<uint32_t*>(host.data() + o_qf);
    auto elem = [&](int r, int k) -> double {
      if (k >= d) return 0.0;
      if (r < dp) return r < d ? cb->pi[(size_t)r * d + k] : 0.0;
      const int i = r - dp;
      return i < L.m ? cb->s[(size_t)i * d + k] : 0.0;
    };
    auto bf_bits = [](double v) -> uint32_t {
      const __nv_bfloat16 h = __double2bfloat16(v);
      return (uint32_t)*reinterpret_cast<const uint16_t*>(&h);
    };
    auto part = [&](double v, int h) -> uint32_t {
      const __nv_bfloat16 hi = __double2bfloat16(v);
      return h == 0 ? bf_bits(v) : bf_bits(v - (double)__bfloat162float(hi));
    };
    for (int mt = 0; mt < R / 16; ++mt)
      for (int j = 0; j < d16; ++j)
        for (int h = 0; h < 2; ++h)
          for (int lane = 0; lane < 32; ++lane) {
            const int g = lane >> 2, t = lane & 3;
            const int r0 = 16 * mt + g, k0 = 16 * j + 2 * t;
            const int rr[4] = {r0, r0 + 8, r0, r0 + 8}, kk[4] = {k0, k0, k0 + 8, k0 + 8};
            uint32_t* dst = qf + ((((size_t)mt * d16 + j) * 2 + h) * 32 + lane) * 4;
            for (int x = 0; x < 4; ++x)
              dst[x] = part(elem(rr[x], kk[x]), h) | (part(elem(rr[x], kk[x] + 1), h) << 16);
          }
  }

  void* dev = nullptr;
  cudaError_t e = cudaMalloc(&dev, total);
  if (e != cudaSuccess) return fail(TQ_ENOMEM, std::string("codebook tables: ") + cudaGetErrorString(e));
  e = cudaMemcpy(dev, host.data(), total, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(dev);
    return cuda_fail(e, "codebook upload");
  }
  uint8_t* base = reinterpret_cast<uint8_t*>(dev);
  cb->dev_block = dev;
  cb->pi32 = reinterpret_cast<float*>(base + o_pi);
  cb->s32 = reinterpret_cast<float*>(base + o_s);
  cb->srott32 = reinterpret_cast<float*>(base + o_srott);
  cb->bound32 = reinterpret_cast<float*>(base + o_b);
  cb->cent32 = reinterpret_cast<float*>(base + o_c);
  cb->pi_bf = reinterpret_cast<__nv_bfloat16*>(base + o_pibf);
  cb->srot_bf = reinterpret_cast<__nv_bfloat16*>(base + o_srbf);
  cb->pit32 = reinterpret_cast<float*>(base + o_pit);
  cb->st32 = reinterpret_cast<float*>(base + o_st);
  cb->qprep_frag = reinterpret_cast<uint4*>(base + o_qf);
  cb->srot32 = reinterpret_cast<float*>(base + o_srot);
  return TQ_OK;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev;
}

int device_sm_count() {
  static int cache[64] = {};
  const int dev = current_device();
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

static tq_status make_view(const tq_codebook* cb, const tq_cache* c, CacheView* v) {
  if (!c) return fail(TQ_EINVAL, "cache is NULL");
  if (!c->pages || !c->block_table) return fail(TQ_EINVAL, "cache pages / block_table is NULL");
  if (!aligned(c->pages, 16)) return fail(TQ_EINVAL, "cache pages must be 16-byte aligned");
  if (!aligned(c->block_table, 4) || (c->error_word && !aligned(c->error_word, 4)))
    return fail(TQ_EINVAL, "cache block_table / error_word must be 4-byte aligned");
  if (c->page_tokens < 16 || c->page_tokens > 256 || (c->page_tokens & (c->page_tokens - 1)) != 0)
    return fail(TQ_EINVAL, "page_tokens must be a power of two in [16, 256]");
  if (c->n_kv_heads < 1 || c->n_pages < 1 || c->max_pages_per_seq < 1)
    return fail(TQ_EINVAL, "cache sizes must be positive");
  v->pages = reinterpret_cast<uint8_t*>(c->pages);
  v->n_pages = c->n_pages;
  v->page_tokens = c->page_tokens;
  v->n_kv_heads = c->n_kv_heads;
  v->block_table = c->block_table;
  v->max_pages = c->max_pages_per_seq;
  v->err = c->error_word;
  v->head_block_bytes = cb->lay.head_block_bytes(c->page_tokens);
  v->page_bytes = v->head_block_bytes * c->n_kv_heads;
  return TQ_OK;
}

static tq_status check_cb(const tq_codebook* cb) {
  if (!cb) return fail(TQ_EINVAL, "codebook is NULL");
  if (!cb->dev_block) return fail(TQ_EINVAL, "codebook has no device tables (host-only build)");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != cb->device) return fail(TQ_EINVAL, "codebook was built for another device");
  return TQ_OK;
}

static size_t dtype_size(tq_dtype dt) { return dt == TQ_F32 ? 4 : 2; }
static bool dtype_ok(tq_dtype dt) { return dt == TQ_BF16 || dt == TQ_F16 || dt == TQ_F32; }

}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_last_error(void) { return g_last_error.c_str(); }

int32_t tq_layout_version(void) { return kLayoutVersion; }

static tq_status build_common(const tq_params* params, tq_codebook** out, bool device) {
  if (!out) return fail(TQ_EINVAL, "out is NULL");
  *out = nullptr;
  tq_status s = check_params(params);
  if (s != TQ_OK) return s;
  tq_codebook* cb = new (std::nothrow) tq_codebook();
  if (!cb) return fail(TQ_ENOMEM, "out of host memory");
  cb->lay = Layout::make(params->d, params->bits, params->m);
  cb->seed_pi = params->seed_pi;
  cb->seed_s = params->seed_s;
  cb->device = -1;
  cb->dev_block = nullptr;
  build_host_tables(cb, params);
  if (device) {
    cudaError_t e = cudaGetDevice(&cb->device);
    if (e != cudaSuccess) {
      delete cb;
      return cuda_fail(e, "cudaGetDevice");
    }
    s = upload(cb);
    if (s != TQ_OK) {
      delete cb;
      return s;
    }
  }
  *out = cb;
  return TQ_OK;
}

tq_status tq_codebook_build(const tq_params* params, tq_codebook** out) {
  return build_common(params, out, true);
}

// Host tables only (no device upload): for inspecting a codebook without a GPU.
tq_status tq_codebook_build_host(const tq_params* params, tq_codebook** out) {
  return build_common(params, out, false);
}

void tq_codebook_free(tq_codebook* cb) {
  if (!cb) return;
  if (cb->dev_block) cudaFree(cb->dev_block);
  delete cb;
}

tq_status tq_codebook_levels(const tq_codebook* cb, double* levels, int32_t* scale_exp) {
  if (!cb || !levels) return fail(TQ_EINVAL, "tq_codebook_levels: codebook / levels is NULL");
  std::memcpy(levels, cb->levels.data(), cb->levels.size() * sizeof(double));
  if (scale_exp) *scale_exp = cb->lay.bits <= 3 ? cb->table_exp : INT32_MIN;
  return TQ_OK;
}

tq_status tq_codebook_export(const tq_codebook* cb, double* pi, double* s, double* centroids,
                             double* boundaries) {
  if (!cb) return fail(TQ_EINVAL, "codebook is NULL");
  if (pi) std::memcpy(pi, cb->pi.data(), cb->pi.size() * sizeof(double));
  if (s && !cb->s.empty()) std::memcpy(s, cb->s.data(), cb->s.size() * sizeof(double));
  if (centroids) std::memcpy(centroids, cb->centroids.data(), cb->centroids.size() * sizeof(double));
  if (boundaries)
    std::memcpy(boundaries, cb->boundaries.data(), cb->boundaries.size() * sizeof(double));
  return TQ_OK;
}

tq_status tq_polar_angle_codebook(int32_t level, int32_t bits, double* centroids, double* boundaries,
                                  double* distortion) {
  if (level < 1 || level > 8) return fail(TQ_EINVAL, "tq_polar_angle_codebook: level must be in [1, 8]");
  if (bits < 1 || bits > 8) return fail(TQ_EUNSUPPORTED, "tq_polar_angle_codebook: bits must be in [1, 8]");
  if (!centroids) return fail(TQ_EINVAL, "tq_polar_angle_codebook: centroids is NULL");
  const tqhost::LloydMax lm = tqhost::polar_angle_lloyd_max(level, bits);
  std::memcpy(centroids, lm.centroids.data(), lm.centroids.size() * sizeof(double));
  if (boundaries) std::memcpy(boundaries, lm.boundaries.data(), lm.boundaries.size() * sizeof(double));
  if (distortion) *distortion = lm.distortion;
  return TQ_OK;
}

tq_status tq_layout(const tq_codebook* cb, int32_t page_tokens, int32_t n_kv_heads,
                    tq_layout_info* info) {
  if (!cb || !info) return fail(TQ_EINVAL, "codebook / info is NULL");
  if (page_tokens < 16 || page_tokens > 256 || (page_tokens & (page_tokens - 1)) != 0 || n_kv_heads < 1)
    return fail(TQ_EINVAL, "page_tokens must be a power of two in [16, 256], n_kv_heads >= 1");
  const Layout& L = cb->lay;
  info->d_pad = L.d_pad;
  info->m_pad = L.m_pad;
  info->words_per_chunk = L.W;
  info->code_bytes = L.code_bytes;
  info->norm_bytes = L.norm_bytes;
  info->head_block_bytes = (int32_t)L.head_block_bytes(page_tokens);
  info->page_bytes = L.head_block_bytes(page_tokens) * n_kv_heads;
  return TQ_OK;
}

tq_status tq_quantize_append(const tq_codebook* cb, const void* x, tq_dtype dtype, int64_t batch,
                             int32_t n_kv_heads, int64_t n_new, const int32_t* start_pos,
                             const tq_cache* cache, void* stream) {
  tq_status s = check_cb(cb);
  if (s != TQ_OK) return s;
  if (!dtype_ok(dtype)) return fail(TQ_EINVAL, "tq_quantize_append: bad dtype");
  if (batch < 0 || n_new < 0) return fail(TQ_EINVAL, "tq_quantize_append: negative size");
  CacheView cv;
  s = make_view(cb, cache, &cv);
  if (s != TQ_OK) return s;
  if (n_kv_heads != cache->n_kv_heads)
    return fail(TQ_EINVAL, "tq_quantize_append: n_kv_heads differs from the cache's");
  if (batch == 0 || n_new == 0) return TQ_OK;
  if (!x || !start_pos) return fail(TQ_EINVAL, "tq_quantize_append: x / start_pos is NULL");
  if (!aligned(x, dtype_size(dtype)) || !aligned(start_pos, 4))
    return fail(TQ_EINVAL, "tq_quantize_append: x / start_pos misaligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bool handled = false;
  s = launch_quantize_tc(cb, x, dtype, batch, n_kv_heads, n_new, start_pos, cv, st, &handled);
  if (handled || s != TQ_OK) return s;
  s = launch_quantize_small(cb, x, dtype, batch, n_kv_heads, n_new, start_pos, cv, st, &handled);
  if (handled || s != TQ_OK) return s;
  return launch_quantize_simt(cb, x, dtype, batch, n_kv_heads, n_new, start_pos, cv, st);
}

tq_status tq_quantize_append_kv(const tq_codebook* key_cb, const void* k, const tq_codebook* value_cb,
                                const void* v, tq_dtype dtype, int64_t batch, int32_t n_kv_heads, int64_t n_new,
                                const int32_t* start_pos, const tq_cache* key_cache, const tq_cache* value_cache,
                                void* stream) {
  tq_status s = check_cb(key_cb);
  if (s != TQ_OK) return s;
  s = check_cb(value_cb);
  if (s != TQ_OK) return s;
  if (!dtype_ok(dtype)) return fail(TQ_EINVAL, "tq_quantize_append_kv: bad dtype");
  if (batch < 0 || n_new < 0) return fail(TQ_EINVAL, "tq_quantize_append_kv: negative size");
  CacheView kv, vv;
  s = make_view(key_cb, key_cache, &kv);
  if (s != TQ_OK) return s;
  s = make_view(value_cb, value_cache, &vv);
  if (s != TQ_OK) return s;
  if (n_kv_heads != key_cache->n_kv_heads || n_kv_heads != value_cache->n_kv_heads)
    return fail(TQ_EINVAL, "tq_quantize_append_kv: n_kv_heads differs from a cache's");
  if (batch == 0 || n_new == 0) return TQ_OK;
  if (!k || !v || !start_pos) return fail(TQ_EINVAL, "tq_quantize_append_kv: NULL pointer");
  if (!aligned(k, dtype_size(dtype)) || !aligned(v, dtype_size(dtype)) || !aligned(start_pos, 4))
    return fail(TQ_EINVAL, "tq_quantize_append_kv: misaligned pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bool handled = false;
  s = launch_quantize_small_kv(key_cb, k, value_cb, v, dtype, batch, n_kv_heads, n_new, start_pos, kv, vv, st,
                               &handled);
  if (handled || s != TQ_OK) return s;
  // other shapes: the two appends one after the other
  s = tq_quantize_append(key_cb, k, dtype, batch, n_kv_heads, n_new, start_pos, key_cache, stream);
  if (s != TQ_OK) return s;
  return tq_quantize_append(value_cb, v, dtype, batch, n_kv_heads, n_new, start_pos, value_cache, stream);
}

size_t tq_logits_workspace_bytes(const tq_codebook* cb, int64_t batch, int32_t n_kv_heads,
                                 int32_t n_q_heads) {
  if (!cb || batch < 0 || n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads)
    return 0;
  return logits_workspace(cb, batch * n_kv_heads, n_q_heads / n_kv_heads);
}

tq_status tq_logits(const tq_codebook* cb, const tq_cache* cache, const void* q, tq_dtype dtype,
                    int64_t batch, int32_t n_q_heads, const int32_t* ctx_len, int64_t max_ctx,
                    float* out, int64_t out_stride, void* workspace, size_t workspace_bytes,
                    void* stream) {
  tq_status s = check_cb(cb);
  if (s != TQ_OK) return s;
  CacheView cv;
  s = make_view(cb, cache, &cv);
  if (s != TQ_OK) return s;
  if (!dtype_ok(dtype)) return fail(TQ_EINVAL, "tq_logits: bad dtype");
  if (batch < 0 || max_ctx < 0 || max_ctx > INT32_MAX) return fail(TQ_EINVAL, "tq_logits: bad size");
  if (n_q_heads < cv.n_kv_heads || n_q_heads % cv.n_kv_heads)
    return fail(TQ_EINVAL, "tq_logits: n_q_heads must be a multiple of the cache's n_kv_heads");
  if (out_stride < max_ctx) return fail(TQ_EINVAL, "tq_logits: out_stride < max_ctx");
  if (max_ctx > cv.max_pages * cv.page_tokens)
    return fail(TQ_EINVAL, "tq_logits: max_ctx exceeds the block table");
  if (batch == 0 || max_ctx == 0) return TQ_OK;
  if (!q || !ctx_len || !out || !workspace) return fail(TQ_EINVAL, "tq_logits: NULL pointer");
  if (!aligned(q, dtype_size(dtype)) || !aligned(out, 4) || !aligned(workspace, 16) || !aligned(ctx_len, 4))
    return fail(TQ_EINVAL, "tq_logits: misaligned pointer");
  return launch_logits(cb, cv, q, dtype, batch, n_q_heads, ctx_len, max_ctx, out, out_stride,
                       workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t tq_logits_topk_workspace_bytes(const tq_codebook* cb, int64_t batch, int32_t n_kv_heads,
                                      int32_t n_q_heads, int64_t max_ctx, int32_t k) {
  if (!cb || batch < 0 || max_ctx < 0 || n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads ||
      k < 1 || k > 32)
    return 0;
  return search_workspace(cb, batch, n_kv_heads, n_q_heads, max_ctx, k);
}

tq_status tq_logits_topk(const tq_codebook* cb, const tq_cache* cache, const void* q, tq_dtype dtype,
                         int64_t batch, int32_t n_q_heads, const int32_t* ctx_len, int64_t max_ctx, int32_t k,
                         float* top_scores, int32_t* top_idx, void* workspace, size_t workspace_bytes,
                         void* stream) {
  tq_status s = check_cb(cb);
  if (s != TQ_OK) return s;
  CacheView cv;
  s = make_view(cb, cache, &cv);
  if (s != TQ_OK) return s;
  if (!dtype_ok(dtype)) return fail(TQ_EINVAL, "tq_logits_topk: bad dtype");
  if (batch < 0 || max_ctx < 0 || max_ctx > INT32_MAX) return fail(TQ_EINVAL, "tq_logits_topk: bad size");
  if (k < 1 || k > 32) return fail(TQ_EINVAL, "tq_logits_topk: k must be in [1, 32]");
  if (n_q_heads < cv.n_kv_heads || n_q_heads % cv.n_kv_heads)
    return fail(TQ_EINVAL, "tq_logits_topk: n_q_heads must be a multiple of the cache's n_kv_heads");
  if (max_ctx > cv.max_pages * cv.page_tokens)
    return fail(TQ_EINVAL, "tq_logits_topk: max_ctx exceeds the block table");
  if (cv.page_tokens < 16) return fail(TQ_EUNSUPPORTED, "tq_logits_topk: pages of fewer than 16 tokens");
  if (batch == 0) return TQ_OK;
  if (!top_scores || !top_idx) return fail(TQ_EINVAL, "tq_logits_topk: NULL pointer");
  if (!aligned(top_scores, 4) || !aligned(top_idx, 4)) return fail(TQ_EINVAL, "tq_logits_topk: misaligned pointer");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (max_ctx == 0) {   // nothing to rank: every entry is (-inf, -1)
    const size_t n = (size_t)batch * n_q_heads * k;
    std::vector<float> hs(n, -INFINITY);
    s = cuda_fail(cudaMemsetAsync(top_idx, 0xFF, n * sizeof(int32_t), st), "tq_logits_topk: clearing idx");
    if (s != TQ_OK) return s;
    return cuda_fail(cudaMemcpyAsync(top_scores, hs.data(), n * sizeof(float), cudaMemcpyHostToDevice, st),
                     "tq_logits_topk: clearing scores");
  }
  if (!q || !ctx_len || !workspace) return fail(TQ_EINVAL, "tq_logits_topk: NULL pointer");
  if (!aligned(q, dtype_size(dtype)) || !aligned(workspace, 256) || !aligned(ctx_len, 4))
    return fail(TQ_EINVAL, "tq_logits_topk: misaligned pointer");
  return launch_search(cb, cv, q, dtype, batch, n_q_heads, ctx_len, max_ctx, k, top_scores, top_idx, workspace,
                       workspace_bytes, st);
}

tq_status tq_polar_build(int32_t d, int32_t bits, int32_t m, uint64_t seed_pi, uint64_t seed_s, tq_polar** out) {
  if (!out) return fail(TQ_EINVAL, "tq_polar_build: out is NULL");
  *out = nullptr;
  if (d != 64 && d != 128 && d != 256) return fail(TQ_EUNSUPPORTED, "tq_polar_build: d must be 64, 128 or 256");
  if (bits < 1 || bits > 4) return fail(TQ_EUNSUPPORTED, "tq_polar_build: bits must be in [1, 4]");
  if (m < 0 || m > d || m % 32) return fail(TQ_EUNSUPPORTED, "tq_polar_build: m must be a multiple of 32 in [0, d]");
  int n_dev = 0;
  if (cudaGetDeviceCount(&n_dev) != cudaSuccess || n_dev == 0) {
    (void)cudaGetLastError();
    return fail(TQ_ECUDA, "tq_polar_build: no CUDA device");
  }
  return polar_build(d, bits, m, seed_pi, seed_s, out);
}

void tq_polar_free(tq_polar* p) { polar_free(p); }

int32_t tq_polar_record_bytes(const tq_polar* p) { return p ? polar_record_bytes(p) : 0; }

tq_status tq_polar_encode(const tq_polar* p, const void* x, tq_dtype dtype, int64_t n, void* records,
                          uint32_t* error_word, void* stream) {
  if (!p) return fail(TQ_EINVAL, "tq_polar_encode: codec is NULL");
  if (!dtype_ok(dtype)) return fail(TQ_EINVAL, "tq_polar_encode: bad dtype");
  if (n < 0) return fail(TQ_EINVAL, "tq_polar_encode: n < 0");
  if (n == 0) return TQ_OK;
  if (!x || !records) return fail(TQ_EINVAL, "tq_polar_encode: NULL pointer");
  if (!aligned(x, dtype_size(dtype)) || !aligned(records, 16) || (error_word && !aligned(error_word, 4)))
    return fail(TQ_EINVAL, "tq_polar_encode: misaligned pointer");
  return polar_encode(p, x, dtype, n, records, error_word, reinterpret_cast<cudaStream_t>(stream));
}

size_t tq_polar_logits_workspace_bytes(const tq_polar* p, int32_t nq) {
  if (!p || nq < 0) return 0;
  return polar_logits_workspace(p, nq);
}

tq_status tq_polar_logits(const tq_polar* p, const void* records, int64_t n, const void* q, tq_dtype dtype,
                          int32_t nq, float* out, int64_t out_stride, void* workspace, size_t workspace_bytes,
                          void* stream) {
  if (!p) return fail(TQ_EINVAL, "tq_polar_logits: codec is NULL");
  if (!dtype_ok(dtype)) return fail(TQ_EINVAL, "tq_polar_logits: bad dtype");
  if (n < 0 || nq < 0 || out_stride < n) return fail(TQ_EINVAL, "tq_polar_logits: bad size");
  if (n == 0 || nq == 0) return TQ_OK;
  if (!records || !q || !out || !workspace) return fail(TQ_EINVAL, "tq_polar_logits: NULL pointer");
  if (!aligned(records, 16) || !aligned(q, dtype_size(dtype)) || !aligned(out, 4) || !aligned(workspace, 16))
    return fail(TQ_EINVAL, "tq_polar_logits: misaligned pointer");
  return polar_logits(p, records, n, q, dtype, nq, out, out_stride, workspace, workspace_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

size_t tq_values_workspace_bytes(const tq_codebook* cb, int64_t batch, int32_t n_kv_heads,
                                 int32_t n_q_heads, int64_t max_ctx) {
  if (!cb || batch < 0 || n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads)
    return 0;
  return values_workspace(cb, batch, n_kv_heads, n_q_heads, max_ctx);
}

tq_status tq_dequant_values(const tq_codebook* cb, const tq_cache* cache, const float* weights,
                            int64_t w_stride, int64_t batch, int32_t n_q_heads,
                            const int32_t* ctx_len, int64_t max_ctx, void* out, tq_dtype out_dtype,
                            int64_t out_stride, void* workspace, size_t workspace_bytes,
                            void* stream) {
  tq_status s = check_cb(cb);
  if (s != TQ_OK) return s;
  CacheView cv;
  s = make_view(cb, cache, &cv);
  if (s != TQ_OK) return s;
  if (!dtype_ok(out_dtype)) return fail(TQ_EINVAL, "tq_dequant_values: bad dtype");
  if (batch < 0 || max_ctx < 0 || max_ctx > INT32_MAX) return fail(TQ_EINVAL, "tq_dequant_values: bad size");
  if (max_ctx > cv.max_pages * cv.page_tokens)
    return fail(TQ_EINVAL, "tq_dequant_values: max_ctx exceeds the block table");
  if (weights) {
    if (out_dtype != TQ_F32) return fail(TQ_EINVAL, "tq_dequant_values: mode B writes fp32");
    if (n_q_heads < cv.n_kv_heads || n_q_heads % cv.n_kv_heads)
      return fail(TQ_EINVAL, "tq_dequant_values: n_q_heads must be a multiple of n_kv_heads");
    if (w_stride < max_ctx) return fail(TQ_EINVAL, "tq_dequant_values: w_stride < max_ctx");
  } else if (out_stride < max_ctx) {
    return fail(TQ_EINVAL, "tq_dequant_values: out_stride < max_ctx");
  }
  if (batch == 0) return TQ_OK;
  if (max_ctx == 0) {
    if (!weights) return TQ_OK;          // mode A: no token to write
    // mode B: every context is empty, so every output row is zero
    if (!out || !aligned(out, 4)) return fail(TQ_EINVAL, "tq_dequant_values: out is NULL or misaligned");
    return cuda_fail(cudaMemsetAsync(out, 0, (size_t)batch * n_q_heads * cb->lay.d * sizeof(float),
                                     reinterpret_cast<cudaStream_t>(stream)),
                     "tq_dequant_values: clearing out");
  }
  if (!ctx_len || !out) return fail(TQ_EINVAL, "tq_dequant_values: NULL pointer");
  if (!aligned(ctx_len, 4)) return fail(TQ_EINVAL, "tq_dequant_values: ctx_len misaligned");
  if (weights && !workspace) return fail(TQ_EINVAL, "tq_dequant_values: mode B needs a workspace");
  const bool misaligned = weights ? !aligned(out, 4) || !aligned(weights, 4) || !aligned(workspace, 4)
                                  : !aligned(out, dtype_size(out_dtype));
  if (misaligned) return fail(TQ_EINVAL, "tq_dequant_values: misaligned pointer");
  return launch_values(cb, cv, weights, w_stride, batch, n_q_heads, ctx_len, max_ctx, out,
                       out_dtype, out_stride, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t tq_attend_workspace_bytes(const tq_codebook* kcb, const tq_codebook* vcb, int64_t batch,
                                 int32_t n_kv_heads, int32_t n_q_heads, int64_t max_ctx) {
  if (!kcb || !vcb || batch < 0 || max_ctx < 0 || n_kv_heads < 1 || n_q_heads < n_kv_heads ||
      n_q_heads % n_kv_heads)
    return 0;
  return attend_workspace(kcb, vcb, batch, n_kv_heads, n_q_heads, max_ctx);
}

tq_status tq_attend(const tq_codebook* kcb, const tq_cache* kcache, const tq_codebook* vcb,
                    const tq_cache* vcache, const void* q, tq_dtype dtype, int64_t batch, int32_t n_q_heads,
                    const int32_t* ctx_len, int64_t max_ctx, float scale, float* out, void* workspace,
                    size_t workspace_bytes, void* stream) {
  tq_status s = check_cb(kcb);
  if (s != TQ_OK) return s;
  s = check_cb(vcb);
  if (s != TQ_OK) return s;
  CacheView kv, vv;
  s = make_view(kcb, kcache, &kv);
  if (s != TQ_OK) return s;
  s = make_view(vcb, vcache, &vv);
  if (s != TQ_OK) return s;
  if (kcb->lay.d != vcb->lay.d) return fail(TQ_EINVAL, "tq_attend: key and value codebooks differ in d");
  if (vcb->lay.m != 0) return fail(TQ_EINVAL, "tq_attend: the value codebook must have m = 0");
  if (kv.n_kv_heads != vv.n_kv_heads) return fail(TQ_EINVAL, "tq_attend: caches differ in n_kv_heads");
  if (!dtype_ok(dtype)) return fail(TQ_EINVAL, "tq_attend: bad dtype");
  if (batch < 0 || max_ctx < 0 || max_ctx > INT32_MAX) return fail(TQ_EINVAL, "tq_attend: bad size");
  if (n_q_heads < kv.n_kv_heads || n_q_heads % kv.n_kv_heads)
    return fail(TQ_EINVAL, "tq_attend: n_q_heads must be a multiple of the caches' n_kv_heads");
  if (max_ctx > kv.max_pages * kv.page_tokens || max_ctx > vv.max_pages * vv.page_tokens)
    return fail(TQ_EINVAL, "tq_attend: max_ctx exceeds a block table");
  if (!std::isfinite(scale)) return fail(TQ_EINVAL, "tq_attend: scale is not finite");
  if (batch == 0) return TQ_OK;
  if (max_ctx == 0) {                    // every context is empty: the rows are zeros
    if (!out || !aligned(out, 4)) return fail(TQ_EINVAL, "tq_attend: out is NULL or misaligned");
    return cuda_fail(cudaMemsetAsync(out, 0, (size_t)batch * n_q_heads * kcb->lay.d * sizeof(float),
                                     reinterpret_cast<cudaStream_t>(stream)),
                     "tq_attend: clearing out");
  }
  if (!q || !ctx_len || !out || !workspace) return fail(TQ_EINVAL, "tq_attend: NULL pointer");
  if (!aligned(q, dtype_size(dtype)) || !aligned(out, 4) || !aligned(workspace, 256) || !aligned(ctx_len, 4))
    return fail(TQ_EINVAL, "tq_attend: misaligned pointer");
  return launch_attend(kcb, kv, vcb, vv, q, dtype, batch, n_q_heads, ctx_len, max_ctx, scale, out, workspace,
                       workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
