// QJL key quantisation: outlier-channel selection, sign sketch, norms.
//
// QJL summary (atlas.scime.ai), Approach: the key is multiplied by a random
// Gaussian JL matrix and only the signs of the result are kept, with the key's
// norm; the outlier channels are sketched apart from the rest. Here the outlier channels of a
// (sequence, kv head) are the n_out channels with the largest energy
// sum_t k_tc^2 over the prefill tokens (outlier channels: "2 numbers out of
// 128 destroy the entire KV cache", section "The Real Problem: Outlier
// Channels"). The inlier sketch sign(S k_in) zeroes those channels; the
// outlier sketch sign(S_out k_out) keeps only them; each part has its norm.
//
// This file holds the CUDA-core path: a channel-energy reduction, a per-head
// top-n selection and a sign-sketch kernel in which one warp owns one token,
// lane j computes sketch row 32r + j and a warp ballot packs the 32 signs of
// word r. Projections run in fp32; a projection whose magnitude is below
// guard * |k_part| is recomputed in fp64, where the bf16 x bf16 (or bf16 x fp32)
// products are exact, so the bit equals the sign of the exact projection.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

template <typename Tin>
__device__ __forceinline__ void load4(const Tin* p, float (&v)[4]);

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
  v[0] = __uint_as_float(w.x << 16);
  v[1] = __uint_as_float(w.x & 0xFFFF0000u);
  v[2] = __uint_as_float(w.y << 16);
  v[3] = __uint_as_float(w.y & 0xFFFF0000u);
}

template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
  const float4 w = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = w.x;
  v[1] = w.y;
  v[2] = w.z;
  v[3] = w.w;
}

// ---------------------------------------------------------------------------
// Channel energy: energy[b, h, c] += sum over a chunk of tokens of k_tc^2 (fp64).
// grid (chunks, Hkv, B), 256 threads; warp w reads tokens chunk_start + w, +8, ...;
// lane l owns channels 4l .. 4l+3 (one 8- or 16-byte load per token).
constexpr int kEnergyChunk = 256;

template <typename Tin>
__global__ void __launch_bounds__(256) channel_energy_kernel(KeysParams p) {
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kEnergyChunk;
  const int t1 = min(p.T, t0 + kEnergyChunk);
  const Tin* base = static_cast<const Tin*>(p.K) + b * p.sb + h * p.sh + 4 * lane;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int t = t0 + warp; t < t1; t += 8) {
    float v[4];
    load4<Tin>(base + t * p.st, v);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] = fma(static_cast<double>(v[k]), static_cast<double>(v[k]), acc[k]);
  }
  __shared__ double red[8][kHeadDim];
#pragma unroll
  for (int k = 0; k < 4; ++k) red[warp][4 * lane + k] = acc[k];
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w][threadIdx.x];
    atomicAdd(p.energy + (static_cast<int64_t>(b) * p.Hkv + h) * kHeadDim + threadIdx.x, s);
  }
}

// ---------------------------------------------------------------------------
// Top-n_out channels per (b, h): repeated warp arg-max, ties to the lower index;
// written in ascending order. One warp per (b, h).
__global__ void __launch_bounds__(32) select_outliers_kernel(KeysParams p) {
  const int bh = blockIdx.x;
  const int lane = threadIdx.x;
  const double* e = p.energy + static_cast<int64_t>(bh) * kHeadDim;
  double v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = e[4 * lane + k];
  uint32_t taken = 0;  // bit k: channel 4*lane+k already chosen
  __shared__ int chosen[kMaxOutliers];
  for (int n = 0; n < p.n_out; ++n) {
    double best = -1.0;
    int best_c = kHeadDim;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (!((taken >> k) & 1u) && v[k] > best) {  // k ascending: first max wins ties
        best = v[k];
        best_c = 4 * lane + k;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oc = __shfl_xor_sync(0xffffffffu, best_c, off);
      if (ob > best || (ob == best && oc < best_c)) {
        best = ob;
        best_c = oc;
      }
    }
    if ((best_c >> 2) == lane) taken |= 1u << (best_c & 3);
    if (lane == 0) chosen[n] = best_c;
  }
  __syncwarp();
  if (lane == 0) {
    for (int i = 1; i < p.n_out; ++i) {  // insertion sort, n_out <= 32
      const int x = chosen[i];
      int j = i - 1;
      while (j >= 0 && chosen[j] > x) {
        chosen[j + 1] = chosen[j];
        --j;
      }
      chosen[j + 1] = x;
    }
  }
  __syncwarp();
  if (lane < p.n_out) p.idx[static_cast<int64_t>(bh) * p.n_out + lane] = chosen[lane];
}

// ---------------------------------------------------------------------------
// Sign sketch. grid (ceil(T / kSketchTokens), Hkv, B), 256 threads (8 warps).
// Shared memory: S^T as bf16 [d][m] (lane-contiguous rows), the outlier matrix
// restricted to the outlier channels as fp32 [n_out][m_out], and per warp the
// masked key k_in (fp32) and the outlier coordinates.
constexpr int kSketchTokens = 64;
constexpr int kSmallT = 32;  // below this many tokens per (b, h) the S^T-from-L2 kernel is used

template <typename Tin>
__global__ void __launch_bounds__(256) sketch_keys_simt_kernel(KeysParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int b = blockIdx.z, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = p.m, m_out = p.m_out, n_out = p.n_out;
  const int wpt = m >> 5;  // words per token (inlier)

  __nv_bfloat16* St = reinterpret_cast<__nv_bfloat16*>(smem_raw);          // [d][m]
  float* So = reinterpret_cast<float*>(St + kHeadDim * m);                   // [n_out][m_out]
  float* kin_s = So + n_out * m_out;                                         // [8][d]
  float* kout_s = kin_s + 8 * kHeadDim;                                      // [8][kMaxOutliers]
  int* idx_s = reinterpret_cast<int*>(kout_s + 8 * kMaxOutliers);            // [n_out]
  unsigned char* is_out = reinterpret_cast<unsigned char*>(idx_s + kMaxOutliers);  // [d]

  const int32_t* idx_g = p.idx + (static_cast<int64_t>(b) * p.Hkv + h) * n_out;
  for (int i = threadIdx.x; i < kHeadDim; i += blockDim.x) is_out[i] = 0;
  __syncthreads();
  if (threadIdx.x < n_out) {
    const int c = min(max(idx_g[threadIdx.x], 0), kHeadDim - 1);  // stay in bounds on bad input
    idx_s[threadIdx.x] = c;
    is_out[c] = 1;
  }
  for (int e = threadIdx.x; e < m * kHeadDim; e += blockDim.x) {
    const int i = e / kHeadDim, c = e % kHeadDim;
    St[c * m + i] = p.S[e];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n_out * m_out; e += blockDim.x) {
    const int o = e / m_out, i = e % m_out;
    So[e] = __bfloat162float(p.S_out[static_cast<int64_t>(i) * kHeadDim + idx_s[o]]);
  }
  __syncthreads();

  const int tb = blockIdx.x * kSketchTokens;
  const int te = min(p.T, tb + kSketchTokens);
  const int pos0 = p.t_start ? p.t_start[b] : 0;
  const Tin* kbase = static_cast<const Tin*>(p.K) + b * p.sb + h * p.sh;
  float* kin = kin_s + warp * kHeadDim;
  float* kout = kout_s + warp * kMaxOutliers;

  for (int t = tb + warp; t < te; t += 8) {
    const int pos = pos0 + t;
    if (pos < 0 || pos >= p.cap) continue;  // warp-uniform
    float v[4];
    load4<Tin>(kbase + t * p.st + 4 * lane, v);
    double nin = 0.0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 4 * lane + k;
      const float x = is_out[c] ? 0.0f : v[k];
      kin[c] = x;
      nin = fma(static_cast<double>(x), static_cast<double>(x), nin);
    }
    __syncwarp();
    double nout = 0.0;
    // outlier coordinates: lane o < n_out fetches channel idx_s[o]
    if (lane < n_out) {
      const int c = idx_s[lane];
      float xo;
      if constexpr (sizeof(Tin) == 2)
        xo = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(kbase)[t * p.st + c]);
      else
        xo = reinterpret_cast<const float*>(kbase)[t * p.st + c];
      kout[lane] = xo;
      nout = static_cast<double>(xo) * static_cast<double>(xo);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      nin += __shfl_xor_sync(0xffffffffu, nin, off);
      nout += __shfl_xor_sync(0xffffffffu, nout, off);
    }
    __syncwarp();
    const double norm_in = sqrt(nin), norm_out = sqrt(nout);
    const float thr_in = p.guard * static_cast<float>(norm_in);
    int j;
    unsigned char* tile = tile_of(p.tiles, p.tl, static_cast<int64_t>(b) * p.Hkv + h, p.cap, pos, &j);
    uint32_t* kbits = reinterpret_cast<uint32_t*>(tile + p.tl.kbits) + j * wpt;

    // inlier sketch: word r collects rows 32r .. 32r+31 (lane j -> row 32r+j)
    uint32_t my_word = 0;
    for (int r = 0; r < wpt; ++r) {
      const int i = 32 * r + lane;
      float y = 0.0f;
#pragma unroll 16
      for (int c = 0; c < kHeadDim; ++c) y = fmaf(__bfloat162float(St[c * m + i]), kin[c], y);
      bool bit = y >= 0.0f;
      if (fabsf(y) < thr_in) {
        double yd = 0.0;
        for (int c = 0; c < kHeadDim; ++c)
          yd = fma(static_cast<double>(__bfloat162float(St[c * m + i])), static_cast<double>(kin[c]), yd);
        bit = yd >= 0.0;
      }
      const uint32_t word = __ballot_sync(0xffffffffu, bit);
      if (lane == r) my_word = word;
    }
    if (lane < wpt) kbits[lane] = my_word;

    // outlier sketch over the n_out outlier coordinates, in fp64 (exact products)
    if (m_out > 0) {
      const int wpo = m_out >> 5;
      uint32_t my_out = 0;
      for (int r = 0; r < wpo; ++r) {
        const int i = 32 * r + lane;
        double yd = 0.0;
        for (int o = 0; o < n_out; ++o)
          yd = fma(static_cast<double>(So[o * m_out + i]), static_cast<double>(kout[o]), yd);
        const uint32_t word = __ballot_sync(0xffffffffu, yd >= 0.0);
        if (lane == r) my_out = word;
      }
      if (lane < wpo) reinterpret_cast<uint32_t*>(tile + p.tl.kbits_out)[j * wpo + lane] = my_out;
    }
    if (lane == 0) {
      __half* kn = reinterpret_cast<__half*>(tile + p.tl.knorm) + 2 * j;
      kn[0] = __double2half(norm_in);
      kn[1] = __double2half(norm_out);
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Sign sketch for a few tokens per (b, h), e.g. the one-token append of a
// decode step. Staging all of S in shared memory would cost more than the
// token itself, so S^T is read from global memory (L2-resident) and the
// d-dimension is split over the 8 warps of a CTA that owns one token: warp w
// sums channels 16w .. 16w+15 for every sketch row (lane l owns rows 8l..8l+7
// of each 256-row pass, one 16-byte load per channel), the partial sums meet
// in shared memory in a fixed order, and thread i finishes row i.
template <typename Tin>
__global__ void __launch_bounds__(256) sketch_keys_small_kernel(KeysParams p) {
  extern __shared__ __align__(16) float red[];  // [8][m]
  __shared__ float kin[kHeadDim];
  __shared__ float kout[kMaxOutliers];
  __shared__ int idx_s[kMaxOutliers];
  __shared__ double nsum[2][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  const int bh = blockIdx.y;
  const int h = bh % p.Hkv, b = bh / p.Hkv;
  const int pos = (p.t_start ? p.t_start[b] : 0) + t;
  if (pos < 0 || pos >= p.cap) return;  // block-uniform
  const int m = p.m, m_out = p.m_out, n_out = p.n_out;
  const int wpt = m >> 5;
  const Tin* krow = static_cast<const Tin*>(p.K) + b * p.sb + h * p.sh + t * p.st;

  if (threadIdx.x < n_out) idx_s[threadIdx.x] = min(max(p.idx[static_cast<int64_t>(bh) * n_out + threadIdx.x], 0), kHeadDim - 1);
  __syncthreads();
  double part_in = 0.0, part_out = 0.0;
  if (threadIdx.x < kHeadDim) {
    const int c = threadIdx.x;
    float x;
    if constexpr (sizeof(Tin) == 2)
      x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(krow)[c]);
    else
      x = reinterpret_cast<const float*>(krow)[c];
    bool out = false;
    for (int o = 0; o < n_out; ++o) out |= idx_s[o] == c;
    kin[c] = out ? 0.0f : x;
    if (out) part_out = static_cast<double>(x) * static_cast<double>(x);
    else part_in = static_cast<double>(x) * static_cast<double>(x);
  }
  if (threadIdx.x < n_out) {
    const int c = idx_s[threadIdx.x];
    float x;
    if constexpr (sizeof(Tin) == 2)
      x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(krow)[c]);
    else
      x = reinterpret_cast<const float*>(krow)[c];
    kout[threadIdx.x] = x;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    part_in += __shfl_xor_sync(0xffffffffu, part_in, off);
    part_out += __shfl_xor_sync(0xffffffffu, part_out, off);
  }
  if (lane == 0) {
    nsum[0][warp] = part_in;
    nsum[1][warp] = part_out;
  }
  __syncthreads();

  // partial projections over this warp's 16 channels
  for (int base = 0; base < m; base += 256) {
    const int row0 = base + 8 * lane;
    if (row0 < m) {
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = 0.0f;
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        const int c = 16 * warp + cc;
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.St + static_cast<int64_t>(c) * m + row0));
        const float kc = kin[c];
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          y[2 * e] = fmaf(__uint_as_float(u[e] << 16), kc, y[2 * e]);
          y[2 * e + 1] = fmaf(__uint_as_float(u[e] & 0xFFFF0000u), kc, y[2 * e + 1]);
        }
      }
      float4* dst = reinterpret_cast<float4*>(red + warp * m + row0);
      dst[0] = make_float4(y[0], y[1], y[2], y[3]);
      dst[1] = make_float4(y[4], y[5], y[6], y[7]);
    }
  }
  __syncthreads();
  double nin = 0.0, nout = 0.0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    nin += nsum[0][w];
    nout += nsum[1][w];
  }
  const double norm_in = sqrt(nin), norm_out = sqrt(nout);
  const float thr = p.guard * static_cast<float>(norm_in);
  int j;
  unsigned char* tile = tile_of(p.tiles, p.tl, bh, p.cap, pos, &j);

  for (int i0 = 0; i0 < m; i0 += 256) {  // m is a multiple of 32: whole warps stay uniform
    const int i = i0 + threadIdx.x;
    if (i0 + 32 * warp < m) {
      float y = 0.0f;
#pragma unroll
      for (int w = 0; w < 8; ++w) y += red[w * m + i];
      bool bit = y >= 0.0f;
      if (fabsf(y) < thr) {
        double yd = 0.0;
        for (int c = 0; c < kHeadDim; ++c)
          yd = fma(static_cast<double>(__bfloat162float(p.St[static_cast<int64_t>(c) * m + i])),
                   static_cast<double>(kin[c]), yd);
        bit = yd >= 0.0;
      }
      const uint32_t word = __ballot_sync(0xffffffffu, bit);
      if (lane == 0) reinterpret_cast<uint32_t*>(tile + p.tl.kbits)[j * wpt + (i >> 5)] = word;
    }
  }
  if (32 * warp < m_out) {  // outlier rows in fp64 over the n_out outlier coordinates (exact products)
    const int i = 32 * warp + lane;
    double yd = 0.0;
    for (int o = 0; o < n_out; ++o)
      yd = fma(static_cast<double>(__bfloat162float(p.S_out[static_cast<int64_t>(i) * kHeadDim + idx_s[o]])),
               static_cast<double>(kout[o]), yd);
    const uint32_t word = __ballot_sync(0xffffffffu, yd >= 0.0);
    if (lane == 0) reinterpret_cast<uint32_t*>(tile + p.tl.kbits_out)[j * (m_out >> 5) + warp] = word;
  }
  if (threadIdx.x == 0) {
    __half* kn = reinterpret_cast<__half*>(tile + p.tl.knorm) + 2 * j;
    kn[0] = __double2half(norm_in);
    kn[1] = __double2half(norm_out);
  }
}

}  // namespace

cudaError_t launch_channel_energy(const KeysParams& p, qjl_dtype dt, cudaStream_t s) {
  dim3 grid((p.T + kEnergyChunk - 1) / kEnergyChunk, p.Hkv, p.B);
  if (dt == QJL_BF16)
    channel_energy_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  else
    channel_energy_kernel<float><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_select_outliers(const KeysParams& p, cudaStream_t s) {
  select_outliers_kernel<<<p.B * p.Hkv, 32, 0, s>>>(p);
  return cudaGetLastError();
}

static size_t sketch_smem_bytes(const KeysParams& p) {
  return static_cast<size_t>(kHeadDim) * p.m * 2 + static_cast<size_t>(p.n_out) * p.m_out * 4 +
         8 * kHeadDim * 4 + 8 * kMaxOutliers * 4 + kMaxOutliers * 4 + kHeadDim;
}

cudaError_t launch_sketch_keys(const KeysParams& p, qjl_dtype dt, cudaStream_t s) {
  if (sketch_keys_tc_applies(p, dt)) return launch_sketch_keys_tc(p, p.num_sms, s);
  if (p.T < kSmallT && static_cast<int64_t>(p.B) * p.Hkv <= 65535) {
    dim3 grid(p.T, p.B * p.Hkv);
    const size_t smem = static_cast<size_t>(8) * p.m * sizeof(float);
    if (dt == QJL_BF16)
      sketch_keys_small_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(p);
    else
      sketch_keys_small_kernel<float><<<grid, 256, smem, s>>>(p);
    return cudaGetLastError();
  }
  const size_t smem = sketch_smem_bytes(p);
  dim3 grid((p.T + kSketchTokens - 1) / kSketchTokens, p.Hkv, p.B);
  const void* fn = dt == QJL_BF16 ? reinterpret_cast<const void*>(sketch_keys_simt_kernel<__nv_bfloat16>)
                                  : reinterpret_cast<const void*>(sketch_keys_simt_kernel<float>);
  cudaError_t e = ensure_smem_limit(fn, smem);
  if (e != cudaSuccess) return e;
  if (dt == QJL_BF16)
    sketch_keys_simt_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(p);
  else
    sketch_keys_simt_kernel<float><<<grid, 256, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace qjl
