// Comparison kernels: decode attention over an unquantised bf16 KV cache, an
// FP8 (E4M3) KV cache and 2- or 4-bit min-max KV caches, and their quantisers.
//
// They give QJL's bandwidth and error trade a baseline on the same harness:
// the exact cache is what the QJL cache replaces ("2 numbers out of 128
// destroy the entire KV cache" (Towards AI), "The Memory Math"), and FP8 is
// the hardware-native halving the TurboQuant slides (section 05, "Why
// Compressing the KV Cache Is Hard") call the easy step. Attention is
// softmax(sm_scale K q) V ("Your Brain Already Runs on 1-Bit Keys", "How
// Attention Computes a Score", "Why Truncation Kills").
//
// FP8 format: E4M3 ("FN": bias 7, 3 mantissa bits, largest finite 448), one
// scale for K and one for V: code = satfinite_rne(fp32(x / scale)) and
// x_hat = code * scale.
// Min-max formats: the token-wise b-bit quantiser of "2 numbers out of 128",
// "The Obvious Fix" (b = 2 or 4, groups of 32 dims, fp16 zero = min and
// scale = (max - min) / (2^b - 1), the code decision of the QJL value codes),
// applied to keys and values alike: the pages' own baseline for a few bits
// per number. A token's row is its codes (dims 8/b per byte, the lowest dim in
// the lowest bits) followed by four (scale, zero) fp16 pairs; x_hat =
// zero + code * scale.
//
// Decode: a (sequence, kv head) pair's tokens are cut into chunks of
// kChunk; one 256-thread block per (chunk, pair) takes all G query heads:
//   1. scores: lane l of a warp owns dims 4l .. 4l+3 of q (pre-scaled by
//      sm_scale log2(e), and k_scale for FP8) and of 8 tokens' keys at a time
//      (each key row read as one coalesced line); the 8 x G
//      partial dots are summed across the warp by a reduce-scatter (halving
//      the values each step), so a token costs about G shuffles;
//   2. per head: the chunk's maximum M and p_t = 2^(x_t - M), L = sum p_t;
//   3. values: every warp accumulates p_t v_t over its tokens (lane l: dims
//      4l .. 4l+3), the warps' sums are added in shared memory;
//   4. the chunk's (o, M, L) go to the workspace, and qjl_merge_partials'
//      kernel combines the chunks (the same exact rescaling).
// Every cache is read once from HBM.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

constexpr int kXWarps = 8;
constexpr int kXThreads = 32 * kXWarps;
constexpr int kChunk = 32 * kXWarps;  // tokens per block: 32 per warp

// 4 dims of a key or value row (lane's dims 4l .. 4l+3) as fp32.
template <int FMT>
__device__ __forceinline__ void load4(const unsigned char* row, int lane, float (&x)[4]);

template <>
__device__ __forceinline__ void load4<QJL_KV_BF16>(const unsigned char* row, int lane, float (&x)[4]) {
  const uint2 w = __ldg(reinterpret_cast<const uint2*>(row) + lane);
  x[0] = __uint_as_float(w.x << 16);
  x[1] = __uint_as_float(w.x & 0xFFFF0000u);
  x[2] = __uint_as_float(w.y << 16);
  x[3] = __uint_as_float(w.y & 0xFFFF0000u);
}

template <>
__device__ __forceinline__ void load4<QJL_KV_FP8_E4M3>(const unsigned char* row, int lane, float (&x)[4]) {
  const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(row) + lane);
  uint32_t h01, h23;  // E4M3 -> f16 is exact
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"(static_cast<unsigned short>(w & 0xFFFFu)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"(static_cast<unsigned short>(w >> 16)));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  x[0] = a.x;
  x[1] = a.y;
  x[2] = b.x;
  x[3] = b.y;
}

// 4 dims of a min-max row: codes of dims 4 lane .. 4 lane + 3 and their group's (scale, zero).
template <int BITS>
__device__ __forceinline__ void load4_minmax(const unsigned char* row, int lane, float (&x)[4]) {
  constexpr int kCodeBytes = kHeadDim * BITS / 8;
  const uint32_t sz = __ldg(reinterpret_cast<const uint32_t*>(row + kCodeBytes) + (lane >> 3));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&sz));  // (scale, zero)
  uint32_t c;
  if constexpr (BITS == 4)
    c = __ldg(reinterpret_cast<const unsigned short*>(row) + lane);
  else
    c = __ldg(row + lane);
#pragma unroll
  for (int k = 0; k < 4; ++k) x[k] = fmaf(static_cast<float>((c >> (BITS * k)) & ((1u << BITS) - 1u)), f.x, f.y);
}

template <>
__device__ __forceinline__ void load4<QJL_KV_MINMAX2>(const unsigned char* row, int lane, float (&x)[4]) {
  load4_minmax<2>(row, lane, x);
}
template <>
__device__ __forceinline__ void load4<QJL_KV_MINMAX4>(const unsigned char* row, int lane, float (&x)[4]) {
  load4_minmax<4>(row, lane, x);
}

__host__ __device__ constexpr int row_bytes_of(int fmt) {
  return fmt == QJL_KV_BF16 ? 2 * kHeadDim
         : fmt == QJL_KV_FP8_E4M3 ? kHeadDim
         : fmt == QJL_KV_MINMAX2 ? kHeadDim / 4 + 16
                                 : kHeadDim / 2 + 16;
}

struct XParams {
  const unsigned char* K;  // [B, Hkv, cap, d] elements of the format
  const unsigned char* V;
  const void* Q;           // [B, Hq, d]
  int q_fp32;
  float k_scale, v_scale;  // FP8 only (1 for bf16)
  int B, Hq, Hkv, cap, T;
  const int32_t* seqlens;
  float sm_scale_log2;
  float* part_o;   // [nchunk][B * Hq][d]
  float* part_ml;  // [nchunk][B * Hq][2]
};

template <int G, int FMT>
__global__ void __launch_bounds__(kXThreads) exact_decode_chunk_kernel(XParams p) {
  constexpr int kRowBytes = row_bytes_of(FMT);
  __shared__ float sc[G][kChunk];                    // logits, then 2^(x - M)
  __shared__ float red[kXWarps][G][kHeadDim];        // the warps' value sums
  __shared__ float ms[G], ls[G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int b = static_cast<int>(bh / p.Hkv), hk = static_cast<int>(bh % p.Hkv);
  int len = p.T;
  if (p.seqlens) len = min(max(p.seqlens[b], 0), p.T);
  const int t0 = chunk * kChunk;
  const int64_t rows = static_cast<int64_t>(p.B) * p.Hq;
  const int64_t row0 = static_cast<int64_t>(b) * p.Hq + hk * G;
  float* po = p.part_o + static_cast<int64_t>(chunk) * rows * kHeadDim;
  float* pml = p.part_ml + static_cast<int64_t>(chunk) * rows * 2;
  if (t0 >= len) {  // an empty chunk: the merge's neutral part
    for (int e = threadIdx.x; e < G * kHeadDim; e += kXThreads) po[row0 * kHeadDim + e] = 0.0f;
    if (threadIdx.x < G) {
      pml[2 * (row0 + threadIdx.x)] = -INFINITY;
      pml[2 * (row0 + threadIdx.x) + 1] = 0.0f;
    }
    return;
  }
  const int n = min(kChunk, len - t0);  // tokens of this chunk
  // ---- q, pre-scaled
  float qf[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const int64_t qo = (row0 + h) * kHeadDim + 4 * lane;
    if (p.q_fp32) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(p.Q) + qo));
      qf[h][0] = v.x; qf[h][1] = v.y; qf[h][2] = v.z; qf[h][3] = v.w;
    } else {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(p.Q) + qo));
      qf[h][0] = __uint_as_float(w.x << 16); qf[h][1] = __uint_as_float(w.x & 0xFFFF0000u);
      qf[h][2] = __uint_as_float(w.y << 16); qf[h][3] = __uint_as_float(w.y & 0xFFFF0000u);
    }
    const float s = p.sm_scale_log2 * p.k_scale;
#pragma unroll
    for (int k = 0; k < 4; ++k) qf[h][k] *= s;
  }
  const unsigned char* Kb = p.K + (bh * p.cap + t0) * static_cast<int64_t>(kRowBytes);
  const unsigned char* Vb = p.V + (bh * p.cap + t0) * static_cast<int64_t>(kRowBytes);
  // ---- 1. logits of this warp's 32 tokens, 8 at a time
#pragma unroll 1
  for (int bt = 0; bt < 4; ++bt) {
    const int tb = 32 * warp + 8 * bt;  // first token of the batch (chunk-relative)
    float a[8][G];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float x[4];
      load4<FMT>(Kb + static_cast<int64_t>(min(tb + k, n - 1)) * kRowBytes, lane, x);
#pragma unroll
      for (int h = 0; h < G; ++h) a[k][h] = fmaf(x[0], qf[h][0], fmaf(x[1], qf[h][1], fmaf(x[2], qf[h][2], x[3] * qf[h][3])));
    }
    // reduce-scatter over the lanes: after the xor-16, -8 and -4 steps lane l
    // holds token (l >> 2) & 7 of the batch, summed over 8 lanes; the xor-2 and
    // -1 steps finish the sum over all 32
    const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4;
    float c4[4][G], c2[2][G], c1[G];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float send = u16 ? a[k][h] : a[k + 4][h], keep = u16 ? a[k + 4][h] : a[k][h];
        c4[k][h] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
      }
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float send = u8 ? c4[k][h] : c4[k + 2][h], keep = u8 ? c4[k + 2][h] : c4[k][h];
        c2[k][h] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
      }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float send = u4 ? c2[0][h] : c2[1][h], keep = u4 ? c2[1][h] : c2[0][h];
      c1[h] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      c1[h] += __shfl_xor_sync(0xffffffffu, c1[h], 2);
      c1[h] += __shfl_xor_sync(0xffffffffu, c1[h], 1);
    }
    if ((lane & 3) == 0) {
      const int t = tb + ((lane >> 2) & 7);
#pragma unroll
      for (int h = 0; h < G; ++h) sc[h][t] = t < n ? c1[h] : -INFINITY;
    }
  }
  __syncthreads();
  // ---- 2. per head (warp h): maximum, weights, sum
  if (warp < G) {
    float M = -INFINITY;
    for (int t = lane; t < kChunk; t += 32) M = fmaxf(M, sc[warp][t]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.0f;
    for (int t = lane; t < kChunk; t += 32) {
      const float w = t < n ? exp2f(sc[warp][t] - M) : 0.0f;
      sc[warp][t] = w;
      L += w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (lane == 0) {
      ms[warp] = M;
      ls[warp] = L;
    }
  }
  __syncthreads();
  // ---- 3. values of this warp's tokens
  float o[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < 4; ++k) o[h][k] = 0.0f;
  const int tw = 32 * warp, tend = min(tw + 32, n);
#pragma unroll 4
  for (int t = tw; t < tend; ++t) {
    float x[4];
    load4<FMT>(Vb + static_cast<int64_t>(t) * kRowBytes, lane, x);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float w = sc[h][t];
#pragma unroll
      for (int k = 0; k < 4; ++k) o[h][k] = fmaf(w, x[k], o[h][k]);
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
    *reinterpret_cast<float4*>(&red[warp][h][4 * lane]) = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
  __syncthreads();
  // ---- 4. the chunk's part
  for (int e = threadIdx.x; e < G * kHeadDim; e += kXThreads) {
    const int h = e / kHeadDim, c = e % kHeadDim;
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kXWarps; ++w) s += red[w][h][c];
    po[(row0 + h) * kHeadDim + c] = s * p.v_scale;
  }
  if (threadIdx.x < G) {
    pml[2 * (row0 + threadIdx.x)] = ms[threadIdx.x];
    pml[2 * (row0 + threadIdx.x) + 1] = ls[threadIdx.x];
  }
}

template <int FMT>
cudaError_t launch_exact_g(const XParams& p, int g, dim3 grid, cudaStream_t s) {
  switch (g) {
    case 1: exact_decode_chunk_kernel<1, FMT><<<grid, kXThreads, 0, s>>>(p); break;
    case 2: exact_decode_chunk_kernel<2, FMT><<<grid, kXThreads, 0, s>>>(p); break;
    case 4: exact_decode_chunk_kernel<4, FMT><<<grid, kXThreads, 0, s>>>(p); break;
    case 8: exact_decode_chunk_kernel<8, FMT><<<grid, kXThreads, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// FP8 quantiser: 8 elements per thread (one 16-byte bf16 load or two fp32
// loads), one 8-byte store of codes.
template <typename Tin>
__global__ void __launch_bounds__(256) fp8_quantize_kernel(const Tin* __restrict__ x, int64_t n8, float scale,
                                                           uint2* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  float v[8];
  if constexpr (sizeof(Tin) == 2) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(x) + i);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __uint_as_float(u[k] << 16);
      v[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
    }
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(x) + 2 * i);
    const float4 b = __ldg(reinterpret_cast<const float4*>(x) + 2 * i + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    unsigned short pr;
    const float lo = __fdiv_rn(v[2 * k], scale), hi = __fdiv_rn(v[2 * k + 1], scale);
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(hi), "f"(lo));
    w[k] = pr;
  }
  out[i] = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// Min-max quantiser: four threads per 32-dim group (8 values each), the
// group's min and max by two shuffles, codes by value_code with 2^BITS - 1
// levels; a thread writes its 8 codes (BITS bytes) and the group's first
// thread the (scale, zero) pair.
template <typename Tin, int BITS>
__global__ void __launch_bounds__(256) minmax_quantize_kernel(const Tin* __restrict__ x, int64_t n_rows,
                                                              unsigned char* __restrict__ out) {
  constexpr int kCodeBytes = kHeadDim * BITS / 8;
  constexpr int kRow = kCodeBytes + 16;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = gid / 16;
  const int chunk = static_cast<int>(gid % 16);  // 8 dims: 8 chunk .. 8 chunk + 7
  const int64_t rr = row < n_rows ? row : n_rows - 1;  // whole 16-lane rows stay in the shuffles
  float v[8];
  if constexpr (sizeof(Tin) == 2) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(x + rr * kHeadDim + 8 * chunk));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __uint_as_float(u[k] << 16);
      v[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
    }
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(x + rr * kHeadDim + 8 * chunk));
    const float4 b = __ldg(reinterpret_cast<const float4*>(x + rr * kHeadDim + 8 * chunk) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  float lo = v[0], hi = v[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    lo = fminf(lo, v[i]);
    hi = fmaxf(hi, v[i]);
  }
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if (row >= n_rows) return;
  constexpr int kTop = (1 << BITS) - 1;
  const __half zero_h = __float2half_rn(lo);
  const __half scale_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), static_cast<float>(kTop)));
  const float zero = __half2float(zero_h), scale = __half2float(scale_h);
  uint32_t word = 0u;
  if (scale != 0.0f) {
    const float rcp = __frcp_rn(scale);
#pragma unroll
    for (int i = 0; i < 8; i += 2) word |= value_code_pair(v[i], v[i + 1], zero, scale, rcp, kTop, BITS) << (BITS * i);
  }
  unsigned char* o = out + row * kRow;
  if constexpr (BITS == 4)
    reinterpret_cast<uint32_t*>(o)[chunk] = word;
  else
    reinterpret_cast<unsigned short*>(o)[chunk] = static_cast<unsigned short>(word);
  if ((chunk & 3) == 0)
    reinterpret_cast<uint32_t*>(o + kCodeBytes)[chunk >> 2] =
        static_cast<uint32_t>(__half_as_ushort(scale_h)) | (static_cast<uint32_t>(__half_as_ushort(zero_h)) << 16);
}

}  // namespace

int exact_row_bytes(int fmt) { return row_bytes_of(fmt); }

cudaError_t launch_minmax_quantize(const void* x, int q_fp32, int64_t n_rows, int bits, unsigned char* out,
                                   cudaStream_t s) {
  const int64_t threads = n_rows * 16;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  const unsigned nb = static_cast<unsigned>(blocks);
  if (q_fp32) {
    if (bits == 2) minmax_quantize_kernel<float, 2><<<nb, 256, 0, s>>>(static_cast<const float*>(x), n_rows, out);
    else minmax_quantize_kernel<float, 4><<<nb, 256, 0, s>>>(static_cast<const float*>(x), n_rows, out);
  } else {
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    if (bits == 2) minmax_quantize_kernel<__nv_bfloat16, 2><<<nb, 256, 0, s>>>(xb, n_rows, out);
    else minmax_quantize_kernel<__nv_bfloat16, 4><<<nb, 256, 0, s>>>(xb, n_rows, out);
  }
  return cudaGetLastError();
}

int64_t exact_decode_chunks(int cap) { return (static_cast<int64_t>(cap) + kChunk - 1) / kChunk; }

cudaError_t launch_exact_decode(int fmt, const void* K, const void* V, float k_scale, float v_scale, int B, int Hq,
                                int Hkv, int cap, int T, const void* Q, int q_fp32, const int32_t* seqlens,
                                float sm_scale_log2, float* O, float* ws, cudaStream_t s) {
  const int64_t nchunk = (static_cast<int64_t>(T) + kChunk - 1) / kChunk;
  const int64_t rows = static_cast<int64_t>(B) * Hq;
  XParams p{};
  p.K = static_cast<const unsigned char*>(K);
  p.V = static_cast<const unsigned char*>(V);
  p.Q = Q;
  p.q_fp32 = q_fp32;
  p.k_scale = fmt == QJL_KV_FP8_E4M3 ? k_scale : 1.0f;
  p.v_scale = fmt == QJL_KV_FP8_E4M3 ? v_scale : 1.0f;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.cap = cap;
  p.T = T;
  p.seqlens = seqlens;
  p.sm_scale_log2 = sm_scale_log2;
  p.part_o = ws;
  p.part_ml = ws + nchunk * rows * kHeadDim;
  if (nchunk > 0x7fffffff || static_cast<int64_t>(B) * Hkv > 65535) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(nchunk), static_cast<unsigned>(B * Hkv));
  const int g = Hq / Hkv;
  cudaError_t e;
  switch (fmt) {
    case QJL_KV_BF16: e = launch_exact_g<QJL_KV_BF16>(p, g, grid, s); break;
    case QJL_KV_FP8_E4M3: e = launch_exact_g<QJL_KV_FP8_E4M3>(p, g, grid, s); break;
    case QJL_KV_MINMAX2: e = launch_exact_g<QJL_KV_MINMAX2>(p, g, grid, s); break;
    case QJL_KV_MINMAX4: e = launch_exact_g<QJL_KV_MINMAX4>(p, g, grid, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_merge_partials(p.part_o, rows * kHeadDim, p.part_ml, 2 * rows, static_cast<int>(nchunk), rows, O, s);
}

cudaError_t launch_fp8_quantize(const void* x, int q_fp32, int64_t n, float scale, unsigned char* out, cudaStream_t s) {
  const int64_t n8 = n / 8;
  const int64_t blocks = (n8 + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (q_fp32)
    fp8_quantize_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, s>>>(static_cast<const float*>(x), n8, scale,
                                                                            reinterpret_cast<uint2*>(out));
  else
    fp8_quantize_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), n8, scale, reinterpret_cast<uint2*>(out));
  return cudaGetLastError();
}

}  // namespace qjl
