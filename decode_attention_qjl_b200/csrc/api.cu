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
  int device;
  int num_sms;
  float guard;
  float row_norm[2];     // max_i |S_i|_2 over the rows of S and of S_out, rounded up
  __nv_bfloat16* S;      // device [m, d] (owns the allocation)
  __nv_bfloat16* St;     // device [d, m], S transposed
  __nv_bfloat16* S_out;  // device [m_out, d] (null when m_out == 0)
  __nv_bfloat16* S_img;   // device [m * d]: S in the tcgen05 B-operand layout
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

// Token splits per (b, kv head) for decode. Work items (one split of one
// (b, kv head)) go round-robin to one persistent CTA per SM, whose NC consumer
// warps share each item's 64-token tiles; a warp also pays a fixed cost per
// item (its query fragments, its partial) of about half a tile. The split count
// minimising (items per CTA) x (tiles per item / NC + 1/2) is taken; each split
// is a whole number of stages (kStageTiles tiles).
void decode_split(const qjl_ctx* ctx, int B, int Hq, int Hkv, int T, int* splits, int* chunk) {
  const int stage = qjl::kStageTiles * qjl::kDecodeTileTokens;
  const int G = Hkv > 0 ? Hq / Hkv : 1;
  const double nc = G <= 2 ? 14.0 : (G == 4 ? 10.0 : 6.0);  // consumer warps per CTA (decode.cu)
  const int64_t n_bh = static_cast<int64_t>(B) * Hkv;
  const int n_stage = T > 0 ? (T + stage - 1) / stage : 1;
  const int max_s = n_stage < 64 ? n_stage : 64;
  double best = -1.0;
  int best_c = n_stage * stage;
  for (int s = 1; s <= max_s; ++s) {
    const int c = (n_stage + s - 1) / s;  // stages per split
    const int s_eff = (n_stage + c - 1) / c;
    if (s_eff != s) continue;  // the same chunk was already tried with fewer splits
    const int64_t per_cta = (n_bh * s + ctx->num_sms - 1) / ctx->num_sms;
    const double cost = static_cast<double>(per_cta) * (c * qjl::kStageTiles / nc + 0.5);
    if (best < 0.0 || cost < best) {
      best = cost;
      best_c = c * stage;
    }
  }
  *chunk = best_c;
  *splits = T > 0 ? (T + best_c - 1) / best_c : 1;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Decode workspace: one merge counter per (sequence, kv head); with several
// splits, the per-split partial results; and the query blocks of the items
// that a CTA cannot keep on chip (past its first kDecodeQBuffers items).
struct DecodeWs {
  size_t tickets, part_o, part_ml, qblock, total;
};

DecodeWs decode_ws_layout(int B, int Hq, int Hkv, int splits, int num_sms, int m, int m_out) {
  DecodeWs w{};
  const size_t bh = static_cast<size_t>(B) * Hkv;
  const int G = Hq / Hkv;
  w.tickets = 0;
  w.total = align256(bh * sizeof(int));
  if (splits > 1) {
    const size_t rows = static_cast<size_t>(B) * Hq * splits;
    w.part_o = w.total;
    w.part_ml = w.part_o + align256(rows * qjl::kHeadDim * sizeof(float));
    w.total = w.part_ml + align256(rows * 2 * sizeof(float));
  }
  const size_t n_items = bh * static_cast<size_t>(splits);
  const size_t grid = n_items < static_cast<size_t>(num_sms) ? n_items : static_cast<size_t>(num_sms);
  const size_t on_chip = static_cast<size_t>(qjl::kDecodeQBuffers) * grid;
  if (n_items > on_chip) {
    w.qblock = w.total;
    w.total += align256((n_items - on_chip) * qjl::decode_qblock_bytes(G, m, m_out));
  }
  return w;
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
  if (!out) return fail(QJL_ERR_ARG, "null output pointer");
  *out = nullptr;
  qjl_status st = check_dims(d, m, m_out, n_outlier);
  if (st != QJL_OK) return st;
  qjl_ctx* ctx = new (std::nothrow) qjl_ctx{};
  if (!ctx) return fail(QJL_ERR_OOM, "host allocation failed");
  ctx->seed = seed;
  ctx->d = d;
  ctx->m = m;
  ctx->m_out = m_out;
  ctx->n_out = n_outlier;
  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device);
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

  // One device allocation: S [m, d], S^T [d, m] (lane-contiguous rows for the
  // small-batch sketch kernel), S_out [m_out, d], S once more in the swizzled
  // layout of the tensor-core sketch's B operand, and S then S_out in the
  // A-fragment order of decode's query projection.
  std::vector<uint16_t> hSt(static_cast<size_t>(m) * d);
  for (int i = 0; i < m; ++i)
    for (int c = 0; c < d; ++c) hSt[static_cast<size_t>(c) * m + i] = hS[static_cast<size_t>(i) * d + c];
  std::vector<uint16_t> hImg(static_cast<size_t>(m) * d), hFrag(static_cast<size_t>(m + m_out) * d);
  qjl::tc_fill_s_image(hS.data(), m, hImg.data());
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

size_t qjl_cache_tile_bytes(int d, int m, int m_out) {
  if (d != qjl::kHeadDim || m < 32 || m > qjl::kMaxM || m % 32 != 0 || m_out < 0 || m_out > qjl::kMaxMOut ||
      m_out % 32 != 0)
    return 0;
  return static_cast<size_t>(qjl::tile_layout(m, m_out).bytes);
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
  p.tl = qjl::tile_layout(ctx->m, ctx->m_out);
  p.energy = static_cast<double*>(workspace);
  p.guard = ctx->guard;
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
  p.tl = qjl::tile_layout(ctx->m, ctx->m_out);
  cudaError_t e = qjl::launch_quantize_values(p, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qjl_quantize_values");
  return QJL_OK;
}

size_t qjl_decode_workspace_bytes(const qjl_ctx* ctx, int B, int Hq, int Hkv, int T) {
  if (!ctx || B < 1 || Hq < 1 || Hkv < 1 || T < 0) return 0;
  int splits, chunk;
  if (Hq % Hkv != 0) return 0;
  decode_split(ctx, B, Hq, Hkv, T, &splits, &chunk);
  return decode_ws_layout(B, Hq, Hkv, splits, ctx->num_sms, ctx->m, ctx->m_out).total;
}

qjl_status qjl_decode_attention(qjl_ctx* ctx, const qjl_cache* cache, const void* Q, qjl_dtype dtype, int Hq,
                                int T, const int32_t* seqlens, float sm_scale, float* O, float* scores,
                                void* workspace, size_t workspace_bytes, void* stream) {
  qjl_status st = check_cache(ctx, cache);
  if (st != QJL_OK) return st;
  if (dtype != QJL_BF16 && dtype != QJL_FP32) return fail(QJL_ERR_ARG, "dtype must be QJL_BF16 or QJL_FP32");
  if (Hq < 1 || Hq % cache->Hkv != 0) return fail(QJL_ERR_ARG, "Hq must be a positive multiple of Hkv");
  const int g = Hq / cache->Hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return fail(QJL_ERR_UNSUPPORTED, "Hq / Hkv must be 1, 2, 4 or 8");
  if (T < 0 || T > cache->cap) return fail(QJL_ERR_ARG, "T must be in [0, cap]");
  if (!Q || !O) return fail(QJL_ERR_ARG, "null Q or O");
  if (!aligned16(Q) || !aligned16(O) || (scores && (reinterpret_cast<uintptr_t>(scores) & 3u)))
    return fail(QJL_ERR_ARG, "Q and O must be 16-byte aligned");
  int splits, chunk;
  decode_split(ctx, cache->B, Hq, cache->Hkv, T, &splits, &chunk);
  const DecodeWs ws = decode_ws_layout(cache->B, Hq, cache->Hkv, splits, ctx->num_sms, ctx->m, ctx->m_out);
  if (!workspace || workspace_bytes < ws.total || !aligned16(workspace))
    return fail(QJL_ERR_WORKSPACE, "qjl_decode_attention: workspace missing, misaligned or too small");

  qjl::DecodeParams p{};
  p.Q = Q;
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
  p.row_norm[0] = ctx->row_norm[0];
  p.row_norm[1] = ctx->row_norm[1];
  p.idx = cache->outlier_idx;
  p.tiles = static_cast<const unsigned char*>(cache->tiles);
  p.tl = qjl::tile_layout(ctx->m, ctx->m_out);
  const float scale = sm_scale > 0.0f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(ctx->d));
  p.sm_scale_log2 = scale * qjl::kLog2e;
  p.O = O;
  p.scores = scores;
  p.splits = splits;
  p.chunk = chunk;
  p.grid = ctx->num_sms;
  char* base = static_cast<char*>(workspace);
  p.tickets = reinterpret_cast<int*>(base + ws.tickets);
  p.qblock = reinterpret_cast<unsigned char*>(base + ws.qblock);
  p.qblock_bytes = static_cast<int>(qjl::decode_qblock_bytes(g, ctx->m, ctx->m_out));
  if (splits > 1) {
    p.part_o = reinterpret_cast<float*>(base + ws.part_o);
    p.part_ml = reinterpret_cast<float*>(base + ws.part_ml);
  }
  cudaError_t e = qjl::launch_decode(p, dtype, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "qjl_decode_attention");
  return QJL_OK;
}

}  // extern "C"
