// C ABI entry points of the QJL library: argument checks, workspace layout and
// kernel launches. Every entry point is declared and documented in qjl.h.
#include <cmath>
#include <limits>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <unordered_map>
#include <vector>

#include "qjl_internal.cuh"

struct qjl_ctx {
  uint64_t seed;
  int d, m, m_out, n_out;
  int vbits;             // value code bits: 4 or 2
  int device;
  int num_sms;
  float guard;
  float guard_tc;        // the tensor-core sketch's band: guard without its 2^-10 floor, over S and S_out
  float row_norm[2];     // max_i |S_i|_2 over the rows of S and of S_out, rounded up
  unsigned long long wait_ns;  // limit of every wait inside the decode kernel
  int clock_khz;               // SM clock rate, to turn the limit into cycles
  __nv_bfloat16* S;      // device [m, d] (owns the allocation)
  __nv_bfloat16* St;     // device [d, m], S transposed
  __nv_bfloat16* S_out;  // device [m_out, d] (null when m_out == 0)
  __nv_bfloat16* S_img;   // device [(m + m_out) * d]: S then S_out in the tcgen05 B-operand layout
  __nv_bfloat16* S_frag;  // device [(m + m_out) * d]: S, S_out in decode's projection A-fragment order
};

namespace {

thread_local std::string g_last_error;

qjl_status fail(qjl_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

qjl_status cuda_fail(cudaError_t e, const char* where) {
  return fail(QJL_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qjl_status check_dims(int d, int m, int m_out, int n_outlier) {
  if (d != qjl::kHeadDim) return fail(QJL_ERR_UNSUPPORTED, "only d = 128 is implemented");
  if (m < 32 || m > qjl::kMaxM || m % 32 != 0) return fail(QJL_ERR_ARG, "m must be a multiple of 32 in [32, 512]");
  if (m_out < 0 || m_out > qjl::kMaxMOut || m_out % 32 != 0)
    return fail(QJL_ERR_ARG, "m_out must be a multiple of 32 in [0, 256]");
  if (n_outlier < 0 || n_outlier > qjl::kMaxOutliers) return fail(QJL_ERR_ARG, "n_outlier must be in [0, 32]");
  if (n_outlier > 0 && m_out == 0) return fail(QJL_ERR_ARG, "n_outlier > 0 needs an outlier sketch (m_out > 0)");
  return QJL_OK;
}

qjl_status check_cache(const qjl_ctx* ctx, const qjl_cache* c) {
  if (!ctx) return fail(QJL_ERR_ARG, "null context");
  if (!c) return fail(QJL_ERR_ARG, "null cache");
  if (c->B < 1 || c->Hkv < 1 || c->cap < 1) return fail(QJL_ERR_ARG, "cache B, Hkv and cap must be >= 1");
  if (c->cap % qjl::kDecodeTileTokens != 0) return fail(QJL_ERR_ARG, "cache cap must be a multiple of 64 tokens");
  if (!c->tiles) return fail(QJL_ERR_ARG, "null cache tiles");
  if (ctx->n_out > 0 && !c->outlier_idx) return fail(QJL_ERR_ARG, "null outlier_idx");
  const void* ptrs[] = {c->outlier_idx, c->tiles};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(QJL_ERR_ARG, "cache arrays must be 16-byte aligned");
  return QJL_OK;
}

qjl_status check_input(const void* X, qjl_dtype dt, int T, int64_t sb, int64_t sh, int64_t st, const char* name) {
  if (dt != QJL_BF16 && dt != QJL_FP32) return fail(QJL_ERR_ARG, "dtype must be QJL_BF16 or QJL_FP32");
  if (T < 0) return fail(QJL_ERR_ARG, "T must be >= 0");
  if (T == 0) return QJL_OK;
  if (!X) return fail(QJL_ERR_ARG, std::string("null ") + name);
  if (!aligned16(X)) return fail(QJL_ERR_ARG, std::string(name) + " must be 16-byte aligned");
  const int64_t q = dt == QJL_BF16 ? 8 : 4;  // elements per 16 bytes
  if (sb < 0 || sh < 0 || st < qjl::kHeadDim || sb % q || sh % q || st % q)
    return fail(QJL_ERR_ARG, std::string(name) + " strides must be non-negative multiples of 16 bytes, stride_t >= d");
  return QJL_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// CTAs of a decode launch: one per SM at most, and no more than the tiles
// the call can have (B * Hkv pairs of up to T tokens each).
int decode_grid(const qjl_ctx* ctx, int B, int Hkv, int T) {
  const int64_t tiles = static_cast<int64_t>(B) * Hkv * ((static_cast<int64_t>(T) + qjl::kDecodeTileTokens - 1) /
                                                         qjl::kDecodeTileTokens);
  return static_cast<int>(tiles < 1 ? 1 : (tiles < ctx->num_sms ? tiles : ctx->num_sms));
}

}  // namespace

namespace qjl {

void set_last_error(const std::string& msg) { g_last_error = msg; }

cudaError_t ensure_smem_limit(const void* func, size_t bytes) {
  static std::mutex mu;
  static std::unordered_map<const void*, size_t> configured;  // per kernel, per process (one device)
  std::lock_guard<std::mutex> lock(mu);
  size_t& cur = configured[func];
  if (bytes <= cur) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) cur = bytes;
  return e;
}

}  // namespace qjl

extern "C" {

const char* qjl_last_error(void) { return g_last_error.c_str(); }

qjl_status qjl_sketch_host(uint64_t seed, int d, int m, int m_out, uint16_t* S, uint16_t* S_out) {
  qjl_status st = check_dims(d, m, m_out, 0);
  if (st != QJL_OK) return st;
  if (!S || (m_out > 0 && !S_out)) return fail(QJL_ERR_ARG, "null output buffer");
  qjl::sketch_fill_host(seed, 0, m, d, S);
  if (m_out > 0) qjl::sketch_fill_host(seed, qjl::kSketchOutOffset, m_out, d, S_out);
  return QJL_OK;
}

qjl_status qjl_init(uint64_t seed, int d, int m, int m_out, int n_outlier, qjl_ctx** out) {
  return qjl_init_ex(seed, d, m, m_out, n_outlier, 4, out);
}

qjl_status qjl_init_ex(uint64_t seed, int d, int m, int m_out, int n_outlier, int value_bits, qjl_ctx** out) {
  if (!out) return fail(QJL_ERR_ARG, "null output pointer");
  *out = nullptr;
  qjl_status st = check_dims(d, m, m_out, n_outlier);
  if (st != QJL_OK) return st;
  if (value_bits != 4 && value_bits != 2) return fail(QJL_ERR_ARG, "value_bits must be 4 or 2");
  qjl_ctx* ctx = new (std::nothrow) qjl_ctx{};
  if (!ctx) return fail(QJL_ERR_OOM, "host allocation failed");
  ctx->vbits = value_bits;
  ctx->seed = seed;
  ctx->d = d;
  ctx->m = m;
  ctx->m_out = m_out;
  ctx->n_out = n_outlier;
  ctx->wait_ns = 2000000000ull;  // 2 s: far beyond any legitimate wait
  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ctx->clock_khz, cudaDevAttrClockRate, ctx->device);
  if (e != cudaSuccess) {
    delete ctx;
    return cuda_fail(e, "qjl_init: device query");
  }
  std::vector<uint16_t> hS(static_cast<size_t>(m) * d), hSo(static_cast<size_t>(m_out) * d);
  qjl::sketch_fill_host(seed, 0, m, d, hS.data());
  if (m_out > 0) qjl::sketch_fill_host(seed, qjl::kSketchOutOffset, m_out, d, hSo.data());

  // Guard band of the fp32 sign decision: a sequential fp32 FMA sum of d exact
  // products has |error| <= d * 2^-24 * sum_c |S_ic k_c| <= d * 2^-24 * |S_i| |k|
  // (Cauchy-Schwarz). The guard is 4x the largest such bound over the rows,
  // and at least 2^-10.
  double max_row = 0.0;
  for (int i = 0; i < m; ++i) {
    double r2 = 0.0;
    for (int c = 0; c < d; ++c) {
      uint32_t u = static_cast<uint32_t>(hS[static_cast<size_t>(i) * d + c]) << 16;
      float f;
      std::memcpy(&f, &u, 4);
      r2 += static_cast<double>(f) * f;
    }
    if (r2 > max_row) max_row = r2;
  }
  const double bound = 4.0 * d * std::ldexp(1.0, -24) * std::sqrt(max_row);
  // Largest row norm of S and of S_out (bf16 values, exact in double), as a
  // float rounded up: |S_i . q| <= row_norm * |q| bounds decode's projections.
  auto max_row_norm = [&](const std::vector<uint16_t>& M, int rows) {
    double best = 0.0;
    for (int i = 0; i < rows; ++i) {
      double r2 = 0.0;
      for (int c = 0; c < d; ++c) {
        uint32_t u = static_cast<uint32_t>(M[static_cast<size_t>(i) * d + c]) << 16;
        float f;
        std::memcpy(&f, &u, 4);
        r2 += static_cast<double>(f) * f;
      }
      best = std::max(best, std::sqrt(r2));
    }
    return std::nextafter(static_cast<float>(best), std::numeric_limits<float>::infinity());
  };
  ctx->row_norm[0] = max_row_norm(hS, m);
  ctx->row_norm[1] = m_out > 0 ? max_row_norm(hSo, m_out) : 0.0f;
  ctx->guard = static_cast<float>(bound > std::ldexp(1.0, -10) ? bound : std::ldexp(1.0, -10));
  // The bulk tensor-core sketch takes the bound itself (4x the sequential
  // round-to-nearest bound, 2x that of a truncating accumulator, over the
  // rows of S and S_out) without the floor: its near-zero entries are
  // recomputed in fp64, and the floor would only add more of them.
  ctx->guard_tc = static_cast<float>(4.0 * d * std::ldexp(1.0, -24) *
                                     std::max(std::sqrt(max_row), static_cast<double>(ctx->row_norm[1])));

  // One device allocation: S [m, d], S^T [d, m] (lane-contiguous rows for the
  // small-batch sketch kernel), S_out [m_out, d], S then S_out once more in the
  // swizzled layout of the tensor-core sketch's B operand, and S then S_out in
  // the A-fragment order of decode's query projection.
  std::vector<uint16_t> hSt(static_cast<size_t>(m) * d);
  for (int i = 0; i < m; ++i)
    for (int c = 0; c < d; ++c) hSt[static_cast<size_t>(c) * m + i] = hS[static_cast<size_t>(i) * d + c];
  std::vector<uint16_t> hImg(static_cast<size_t>(m + m_out) * d), hFrag(static_cast<size_t>(m + m_out) * d);
  {
    std::vector<uint16_t> both(hS);
    both.insert(both.end(), hSo.begin(), hSo.end());
    qjl::tc_fill_s_image(both.data(), m + m_out, hImg.data());
  }
  qjl::decode_fill_s_frag(hS.data(), hSo.data(), m, m_out, hFrag.data());
  const size_t n_all = hS.size() + hSt.size() + hSo.size() + hImg.size() + hFrag.size();
  e = cudaMalloc(&ctx->S, n_all * sizeof(uint16_t));
  if (e != cudaSuccess) {
    delete ctx;
    return fail(QJL_ERR_OOM, std::string("qjl_init: cudaMalloc: ") + cudaGetErrorString(e));
  }
  ctx->St = ctx->S + hS.size();
  ctx->S_out = m_out > 0 ? ctx->St + hSt.size() : nullptr;
  ctx->S_img = ctx->St + hSt.size() + hSo.size();  // 16-byte aligned: every part is a multiple of d bf16
  ctx->S_frag = ctx->S_img + hImg.size();
  e = cudaMemcpy(ctx->S, hS.data(), hS.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(ctx->S_img, hImg.data(), hImg.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(ctx->S_frag, hFrag.data(), hFrag.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(ctx->St, hSt.data(), hSt.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && m_out > 0)
    e = cudaMemcpy(ctx->S_out, hSo.data(), hSo.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaFree(ctx->S);
    delete ctx;
    return cuda_fail(e, "qjl_init: upload");
  }
  *out = ctx;
  return QJL_OK;
}

void qjl_free(qjl_ctx* ctx) {
  if (!ctx) return;
  cudaDeviceSynchronize();
  cudaFree(ctx->S);  // S, S^T and S_out share one allocation
  delete ctx;
}

qjl_status qjl_ctx_sketch(const qjl_ctx* ctx, uint16_t* S, uint16_t* S_out) {
  if (!ctx || !S || (ctx->m_out > 0 && !S_out)) return fail(QJL_ERR_ARG, "null argument");
  cudaError_t e = cudaMemcpy(S, ctx->S, static_cast<size_t>(ctx->m) * ctx->d * 2, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && ctx->m_out > 0)
    e = cudaMemcpy(S_out, ctx->S_out, static_cast<size_t>(ctx->m_out) * ctx->d * 2, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "qjl_ctx_sketch");
  return QJL_OK;
}

float qjl_ctx_guard(const qjl_ctx* ctx) { return ctx ? ctx->guard : 0.0f; }

size_t qjl_cache_tile_bytes(int d, int m, int m_out) { return qjl_cache_tile_bytes_ex(d, m, m_out, 4); }

size_t qjl_cache_tile_bytes_ex(int d, int m, int m_out, int value_bits) {
  if (d != qjl::kHeadDim || m < 32 || m > qjl::kMaxM || m % 32 != 0 || m_out < 0 || m_out > qjl::kMaxMOut ||
      m_out % 32 != 0 || (value_bits != 4 && value_bits != 2))
    return 0;
  return static_cast<size_t>(qjl::tile_layout(m, m_out, value_bits).bytes);
}

size_t qjl_quantize_keys_workspace_bytes(const qjl_ctx* ctx, int B, int Hkv, qjl_mode mode) {
  (void)ctx;
  if (mode != QJL_PREFILL || B < 1 || Hkv < 1) return 0;
  return align256(static_cast<size_t>(B) * Hkv * qjl::kHeadDim * sizeof(double));
}

qjl_status qjl_quantize_keys(qjl_ctx* ctx, const qjl_cache* cache, const void* K, qjl_dtype dtype, int T,
                             int64_t stride_b, int64_t stride_h, int64_t stride_t, const int32_t* t_start,
                             qjl_mode mode, void* workspace, size_t workspace_bytes, void* stream) {
  qjl_status st = check_cache(ctx, cache);
  if (st != QJL_OK) return st;
  st = check_input(K, dtype, T, stride_b, stride_h, stride_t, "K");
  if (st != QJL_OK) return st;
  if (mode != QJL_PREFILL && mode != QJL_APPEND) return fail(QJL_ERR_ARG, "mode must be QJL_PREFILL or QJL_APPEND");
  if (!t_start && T > cache->cap) return fail(QJL_ERR_ARG, "T exceeds the cache capacity");
  if (T == 0) return QJL_OK;
  const bool select = mode == QJL_PREFILL && ctx->n_out > 0;
  const size_t need = select ? qjl_quantize_keys_workspace_bytes(ctx, cache->B, cache->Hkv, mode) : 0;
  if (select && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(QJL_ERR_WORKSPACE, "qjl_quantize_keys: workspace missing, misaligned or too small");

  qjl::KeysParams p{};
  p.K = K;
  p.sb = stride_b;
  p.sh = stride_h;
  p.st = stride_t;
  p.B = cache->B;
  p.Hkv = cache->Hkv;
  p.T = T;
  p.cap = cache->cap;
  p.t_start = t_start;
  p.m = ctx->m;
  p.m_out = ctx->m_out;
  p.n_out = ctx->n_out;
  p.S = ctx->S;
  p.St = ctx->St;
  p.S_out = ctx->S_out;
  p.idx = cache->outlier_idx;
  p.tiles = static_cast<unsigned char*>(cache->tiles);
  p.tl = qjl::tile_layout(ctx->m, ctx->m_out, ctx->vbits);
  p.energy = static_cast<double*>(workspace);
  p.guard = ctx->guard;
  p.guard_tc = ctx->guard_tc;
  p.S_img = ctx->S_img;
  p.num_sms = ctx->num_sms;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (select) {
    e = cudaMemsetAsync(workspace, 0, need, s);
    if (e != cudaSuccess) return cuda_fail(e, "qjl_quantize_keys: memset");
    e = qjl::launch_channel_energy(p, dtype, s);
    if (e != cudaSuccess) return cuda_fail(e, "qjl_quantize_keys: channel energy");
    e = qjl::launch_select_outliers(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "qjl_quantize_keys: select");
  }
  e = qjl::launch_sketch_keys(p, dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "qjl_quantize_keys: sketch");
  return QJL_OK;
}

qjl_status qjl_quantize_values(qjl_ctx* ctx, const qjl_cache* cache, const void* V, qjl_dtype dtype, int T,
                               int64_t stride_b, int64_t stride_h, int64_t stride_t, const int32_t* t_start,
                               void* stream) {
  qjl_status st = check_cache(ctx, cache);
  if (st != QJL_OK) return st;
  st = check_input(V, dtype, T, stride_b, stride_h, stride_t, "V");
  if (st != QJL_OK) return st;
  if (!t_start && T > cache->cap) return fail(QJL_ERR_ARG, "T exceeds the cache capacity");
  if (static_cast<int64_t>(cache->B) * cache->Hkv > 65535)
    return fail(QJL_ERR_UNSUPPORTED, "B * Hkv must be at most 65535");
  if (T == 0) return QJL_OK;
  qjl::ValuesParams p{};
  p.V = V;
  p.sb = stride_b;
  p.sh = stride_h;
  p.st = stride_t;
  p.B = cache->B;
  p.Hkv = cache->Hkv;
  p.T = T;
  p.cap = cache->cap;
  p.t_start = t_start;
  p.tiles = static_cast<unsigned char*>(cache->tiles);
  p.tl = qjl::tile_layout(ctx->m, ctx->m_out, ctx->vbits);
  cudaError_t e = qjl::launch_quantize_values(p, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qjl_quantize_values");
  return QJL_OK;
}

size_t qjl_decode_workspace_bytes(const qjl_ctx* ctx, int B, int Hq, int Hkv, int T) {
  if (!ctx || B < 1 || Hq < 1 || Hkv < 1 || T < 0 || Hq % Hkv != 0) return 0;
  return qjl::decode_ws_layout(B, Hq, Hkv, ctx->num_sms, ctx->m, ctx->m_out).total;
}

}  // extern "C"

namespace {

// Shared by qjl_decode_attention and qjl_decode_step: checks, workspace
// layout and the launch. K_new / V_new are null for qjl_decode_attention.
qjl_status decode_common(const char* fn, qjl_ctx* ctx, const qjl_cache* cache, const void* Q, const void* K_new,
                         int64_t k_sb, int64_t k_sh, const void* V_new, int64_t v_sb, int64_t v_sh,
                         qjl_dtype dtype, int Hq, int T, const int32_t* seqlens, float sm_scale, float* O,
                         float* ML, float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  qjl_status st = check_cache(ctx, cache);
  if (st != QJL_OK) return st;
  if (dtype != QJL_BF16 && dtype != QJL_FP32) return fail(QJL_ERR_ARG, "dtype must be QJL_BF16 or QJL_FP32");
  if (Hq < 1 || Hq % cache->Hkv != 0) return fail(QJL_ERR_ARG, "Hq must be a positive multiple of Hkv");
  const int g = Hq / cache->Hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return fail(QJL_ERR_UNSUPPORTED, "Hq / Hkv must be 1, 2, 4 or 8");
  const bool append = K_new != nullptr;
  if (T < 0 || T + (append ? 1 : 0) > cache->cap)
    return fail(QJL_ERR_ARG, append ? "T must be in [0, cap - 1] (the appended token needs a slot)"
                                    : "T must be in [0, cap]");
  if (!Q || !O) return fail(QJL_ERR_ARG, "null Q or O");
  if (!aligned16(Q) || !aligned16(O) || (scores && (reinterpret_cast<uintptr_t>(scores) & 3u)))
    return fail(QJL_ERR_ARG, "Q and O must be 16-byte aligned");
  if (ML && (reinterpret_cast<uintptr_t>(ML) & 7u)) return fail(QJL_ERR_ARG, "ML must be 8-byte aligned");
  if (append) {
    if (!V_new) return fail(QJL_ERR_ARG, "null V_new");
    const int64_t q = dtype == QJL_BF16 ? 8 : 4;  // elements per 16 bytes
    if (!aligned16(K_new) || !aligned16(V_new) || k_sb < 0 || k_sh < 0 || v_sb < 0 || v_sh < 0 || k_sb % q ||
        k_sh % q || v_sb % q || v_sh % q)
      return fail(QJL_ERR_ARG, "K_new and V_new must be 16-byte aligned with strides of whole 16-byte units");
  }
  const qjl::DecodeWsLayout ws = qjl::decode_ws_layout(cache->B, Hq, cache->Hkv, ctx->num_sms, ctx->m, ctx->m_out);
  if (!workspace || workspace_bytes < ws.total || !aligned16(workspace))
    return fail(QJL_ERR_WORKSPACE, std::string(fn) + ": workspace missing, misaligned or too small");

  qjl::DecodeParams p{};
  p.Q = Q;
  p.K_new = K_new;
  p.V_new = V_new;
  p.k_sb = k_sb;
  p.k_sh = k_sh;
  p.v_sb = v_sb;
  p.v_sh = v_sh;
  p.append = append ? 1 : 0;
  p.B = cache->B;
  p.Hq = Hq;
  p.Hkv = cache->Hkv;
  p.T = T;
  p.cap = cache->cap;
  p.seqlens = seqlens;
  p.m = ctx->m;
  p.m_out = ctx->m_out;
  p.n_out = ctx->n_out;
  p.S = ctx->S;
  p.S_out = ctx->S_out;
  p.S_frag = reinterpret_cast<const uint4*>(ctx->S_frag);
  // the tensor-core sums have no specified order: twice the sequential-sum guard band
  p.guard = 2.0f * ctx->guard;
  p.idx = cache->outlier_idx;
  p.tiles = static_cast<unsigned char*>(cache->tiles);
  p.tl = qjl::tile_layout(ctx->m, ctx->m_out, ctx->vbits);
  const float scale = sm_scale > 0.0f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(ctx->d));
  p.sm_scale_log2 = scale * qjl::kLog2e;
  p.O = O;
  p.ML = ML;
  p.scores = scores;
  p.score_stride = T + p.append;
  p.grid = decode_grid(ctx, cache->B, cache->Hkv, T + p.append);
  char* base = static_cast<char*>(workspace);
  p.hdr = reinterpret_cast<int*>(base + ws.hdr);
  p.tickets = reinterpret_cast<int*>(base + ws.tickets);
  p.qblock = reinterpret_cast<unsigned char*>(base + ws.qblock);
  p.qblock_bytes = static_cast<int>(qjl::decode_qblock_bytes(g, ctx->m, ctx->m_out));
  p.part_o = reinterpret_cast<float*>(base + ws.part_o);
  p.part_ml = reinterpret_cast<float*>(base + ws.part_ml);
  // limit in cycles at the maximum SM clock (a lower clock only makes the wait longer in time)
  p.wait_cycles = ctx->wait_ns * static_cast<unsigned long long>(ctx->clock_khz > 0 ? ctx->clock_khz : 2000000) / 1000000ull;
  if (p.wait_cycles == 0) p.wait_cycles = 1;
  cudaError_t e = qjl::launch_decode(p, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return QJL_OK;
}

}  // namespace

namespace qjl {

size_t decode_ws_zero_bytes(const qjl_ctx* ctx, int B, int Hq, int Hkv) {
  if (!ctx || B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return 0;
  return decode_ws_layout(B, Hq, Hkv, ctx->num_sms, ctx->m, ctx->m_out).zero_bytes;
}

int ctx_device(const qjl_ctx* ctx) { return ctx ? ctx->device : -1; }

}  // namespace qjl

extern "C" {

qjl_status qjl_decode_attention(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, qjl_dtype dtype, int Hq,
                                int T, const int32_t* seqlens, float sm_scale, float* O, float* scores,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return decode_common("qjl_decode_attention", ctx, cache, Q, nullptr, 0, 0, nullptr, 0, 0, dtype, Hq, T, seqlens,
                       sm_scale, O, nullptr, scores, workspace, workspace_bytes, stream);
}

qjl_status qjl_decode_attention_partial(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, qjl_dtype dtype, int Hq,
                                        int T, const int32_t* seqlens, float sm_scale, float* O_part, float* ML_part,
                                        float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (!ML_part) return fail(QJL_ERR_ARG, "qjl_decode_attention_partial: null ML_part");
  return decode_common("qjl_decode_attention_partial", ctx, cache, Q, nullptr, 0, 0, nullptr, 0, 0, dtype, Hq, T,
                       seqlens, sm_scale, O_part, ML_part, scores, workspace, workspace_bytes, stream);
}

qjl_status qjl_merge_partials(const float* O_parts, int64_t o_stride, const float* ML_parts, int64_t ml_stride, int R,
                              int64_t rows, float* O, void* stream) {
  if (R < 1 || rows < 0) return fail(QJL_ERR_ARG, "qjl_merge_partials: R must be >= 1 and rows >= 0");
  if (rows == 0) return QJL_OK;
  if (!O_parts || !ML_parts || !O) return fail(QJL_ERR_ARG, "qjl_merge_partials: null buffer");
  if (R > 1 && (o_stride < rows * qjl::kHeadDim || ml_stride < 2 * rows))
    return fail(QJL_ERR_ARG, "qjl_merge_partials: rank strides smaller than one rank's parts");
  if (!aligned16(O_parts) || !aligned16(O) || (reinterpret_cast<uintptr_t>(ML_parts) & 7u) || o_stride % 4 != 0 ||
      ml_stride % 2 != 0)
    return fail(QJL_ERR_ARG, "qjl_merge_partials: O_parts (and its rank stride) and O must be 16-byte aligned, "
                             "ML_parts (and its stride) 8-byte aligned");
  cudaError_t e = qjl::launch_merge_partials(O_parts, o_stride, ML_parts, ml_stride, R, rows, O,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qjl_merge_partials");
  return QJL_OK;
}

qjl_status qjl_decode_step(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, const void* K_new, int64_t k_stride_b,
                           int64_t k_stride_h, const void* V_new, int64_t v_stride_b, int64_t v_stride_h,
                           qjl_dtype dtype, int Hq, int T, const int32_t* seqlens, float sm_scale, float* O,
                           float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (!K_new) return fail(QJL_ERR_ARG, "qjl_decode_step: null K_new");
  return decode_common("qjl_decode_step", ctx, cache, Q, K_new, k_stride_b, k_stride_h, V_new, v_stride_b,
                       v_stride_h, dtype, Hq, T, seqlens, sm_scale, O, nullptr, scores, workspace, workspace_bytes,
                       stream);
}

qjl_status qjl_fp8_quantize(const void* X, qjl_dtype dtype, int64_t n, float scale, uint8_t* out, void* stream) {
  if (n < 0 || n % 8 != 0) return fail(QJL_ERR_ARG, "qjl_fp8_quantize: n must be a non-negative multiple of 8");
  if (!(scale > 0.0f) || !std::isfinite(scale)) return fail(QJL_ERR_ARG, "qjl_fp8_quantize: scale must be > 0");
  if (dtype != QJL_BF16 && dtype != QJL_FP32) return fail(QJL_ERR_ARG, "qjl_fp8_quantize: dtype");
  if (n == 0) return QJL_OK;
  if (!X || !out || !aligned16(X) || (reinterpret_cast<uintptr_t>(out) & 7u))
    return fail(QJL_ERR_ARG, "qjl_fp8_quantize: X must be 16-byte and out 8-byte aligned");
  cudaError_t e = qjl::launch_fp8_quantize(X, dtype == QJL_FP32, n, scale, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qjl_fp8_quantize");
  return QJL_OK;
}

qjl_status qjl_minmax_quantize(const void* X, qjl_dtype dtype, int64_t n_rows, int bits, uint8_t* out, void* stream) {
  if (n_rows < 0 || (bits != 2 && bits != 4)) return fail(QJL_ERR_ARG, "qjl_minmax_quantize: n_rows >= 0, bits 2 or 4");
  if (dtype != QJL_BF16 && dtype != QJL_FP32) return fail(QJL_ERR_ARG, "qjl_minmax_quantize: dtype");
  if (n_rows == 0) return QJL_OK;
  if (!X || !out || !aligned16(X) || !aligned16(out))
    return fail(QJL_ERR_ARG, "qjl_minmax_quantize: X and out must be 16-byte aligned");
  cudaError_t e = qjl::launch_minmax_quantize(X, dtype == QJL_FP32, n_rows, bits, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qjl_minmax_quantize");
  return QJL_OK;
}

size_t qjl_exact_decode_workspace_bytes(int B, int Hq, int T) {
  if (B < 1 || Hq < 1 || T < 0) return 0;
  const int64_t rows = static_cast<int64_t>(B) * Hq;
  return static_cast<size_t>(qjl::exact_decode_chunks(T) * rows * (qjl::kHeadDim + 2) * 4);
}

qjl_status qjl_exact_decode(qjl_kv_format format, const void* K, const void* V, float k_scale, float v_scale, int B,
                            int Hq, int Hkv, int cap, int T, const void* Q, qjl_dtype q_dtype,
                            const int32_t* seqlens, float sm_scale, float* O, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (format != QJL_KV_BF16 && format != QJL_KV_FP8_E4M3 && format != QJL_KV_MINMAX2 && format != QJL_KV_MINMAX4)
    return fail(QJL_ERR_ARG, "qjl_exact_decode: format");
  if (q_dtype != QJL_BF16 && q_dtype != QJL_FP32) return fail(QJL_ERR_ARG, "qjl_exact_decode: q_dtype");
  if (B < 1 || Hkv < 1 || Hq < 1 || Hq % Hkv != 0 || T < 0 || T > cap || B * static_cast<int64_t>(Hkv) > 65535)
    return fail(QJL_ERR_ARG, "qjl_exact_decode: shapes (B, Hq, Hkv, cap, T)");
  const int g = Hq / Hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return fail(QJL_ERR_UNSUPPORTED, "qjl_exact_decode: Hq / Hkv");
  if (format == QJL_KV_FP8_E4M3 && (!(k_scale > 0.0f) || !(v_scale > 0.0f)))
    return fail(QJL_ERR_ARG, "qjl_exact_decode: FP8 scales must be > 0");
  if (!K || !V || !Q || !O || !aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(O))
    return fail(QJL_ERR_ARG, "qjl_exact_decode: null or misaligned K, V, Q or O");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(O, 0, static_cast<size_t>(B) * Hq * qjl::kHeadDim * 4, s);
    return e == cudaSuccess ? QJL_OK : cuda_fail(e, "qjl_exact_decode");
  }
  if (!workspace || !aligned16(workspace) || workspace_bytes < qjl_exact_decode_workspace_bytes(B, Hq, T))
    return fail(QJL_ERR_WORKSPACE, "qjl_exact_decode: workspace missing, misaligned or too small");
  const float scale = sm_scale > 0.0f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(qjl::kHeadDim));
  cudaError_t e = qjl::launch_exact_decode(format, K, V, k_scale, v_scale, B, Hq, Hkv, cap, T, Q,
                                           q_dtype == QJL_FP32, seqlens, scale * qjl::kLog2e, O,
                                           static_cast<float*>(workspace), s);
  if (e != cudaSuccess) return cuda_fail(e, "qjl_exact_decode");
  return QJL_OK;
}

qjl_status qjl_set_wait_limit(qjl_ctx* ctx, uint64_t ns) {
  if (!ctx || ns == 0) return fail(QJL_ERR_ARG, "qjl_set_wait_limit: null context or zero limit");
  ctx->wait_ns = ns;
  return QJL_OK;
}

qjl_status qjl_decode_workspace_status(const qjl_ctx* ctx, void* workspace, int B, int Hq, int Hkv, void* stream) {
  if (!ctx || !workspace) return fail(QJL_ERR_ARG, "qjl_decode_workspace_status: null context or workspace");
  const size_t zero = qjl::decode_ws_zero_bytes(ctx, B, Hq, Hkv);
  if (zero == 0) return fail(QJL_ERR_ARG, "qjl_decode_workspace_status: invalid shape");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int hdr[3] = {0, 0, 0};
  cudaError_t e = cudaMemcpyAsync(hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "qjl_decode_workspace_status");
  if ((hdr[2] & qjl::kDecodeErrTimeout) == 0) return QJL_OK;
  // a wait ran out: counters may be left mid-call; clear them for the next call
  e = cudaMemsetAsync(workspace, 0, zero, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "qjl_decode_workspace_status: clear");
  return fail(QJL_ERR_TIMEOUT, "a wait inside the decode kernel ran out (its outputs hold NaN); "
                               "the workspace counters were cleared");
}

}  // extern "C"
