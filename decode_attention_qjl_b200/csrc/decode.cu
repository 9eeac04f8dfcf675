// QJL decode attention, CUDA-core path (one kernel launch per call).
//
// For each sequence b and kv head hk, the G = Hq/Hkv query heads that share the
// head are processed together (grouped-query attention, contiguous groups).
// QJL summary (atlas.scime.ai), Approach: the query is JL-projected WITHOUT
// quantisation, and a cached token's score is the asymmetric estimator
//   s_t = sqrt(pi/2)/m * |k_in| * <S q_in, sign(S k_in)>
//       + sqrt(pi/2)/m_out * |k_out| * <S_out q_out, sign(S_out k_out)>.
// With packed bits, <sq, sign> = 2 * sum_{bit set} sq_i - sum_i sq_i.
// Softmax is online (running max and sum) and the value accumulation reads the
// 4-bit codes with their fp16 scale and zero.
//
// Work split: grid (splits, Hkv, B), 256 threads. Each CTA projects the query
// into shared memory, then each warp scores 32 tokens at a time (lane = token),
// updates its own running max/sum, and accumulates p_t * v_t with lane l
// owning dims 4l..4l+3. Warps combine in shared memory; with several splits the
// CTA writes an unnormalised partial (max, sum, o) and the last CTA of the
// (b, hk) group, found with an atomic ticket, merges them (no spin-waits).
#include "qjl_internal.cuh"

namespace qjl {
namespace {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeWarps = kDecodeThreads / 32;

template <typename Tq>
__device__ __forceinline__ float load_q(const Tq* q, int i);
template <>
__device__ __forceinline__ float load_q<__nv_bfloat16>(const __nv_bfloat16* q, int i) {
  return __bfloat162float(q[i]);
}
template <>
__device__ __forceinline__ float load_q<float>(const float* q, int i) {
  return q[i];
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

template <int G, typename Tq>
__global__ void __launch_bounds__(kDecodeThreads) decode_simt_kernel(DecodeParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = p.m, m_out = p.m_out, n_out = p.n_out;
  int len = p.seqlens ? p.seqlens[b] : p.T;
  len = max(0, min(len, p.T));
  const int t0 = split * p.chunk;
  const int t1 = min(len, t0 + p.chunk);

  float* sq_in = reinterpret_cast<float*>(smem_raw);  // [G][m]
  float* sq_out = sq_in + G * m;                        // [G][m_out]
  float* q_in = sq_out + G * m_out;                     // [G][d], outlier channels zeroed
  float* q_out = q_in + G * kHeadDim;                   // [G][kMaxOutliers]
  float* red = q_out + G * kMaxOutliers;                // [warps][G][d]
  float* wm = red + kDecodeWarps * G * kHeadDim;        // [warps][G]
  float* wl = wm + kDecodeWarps * G;                    // [warps][G]
  float* sums = wl + kDecodeWarps * G;                  // [G][2]
  int* idx_s = reinterpret_cast<int*>(sums + 2 * G);    // [kMaxOutliers]
  int* flag = idx_s + kMaxOutliers;                     // [1]
  unsigned char* is_out = reinterpret_cast<unsigned char*>(flag + 1);  // [d]

  // ---- query projection: sq_in = S q_in, sq_out = S_out q_out (fp32) ----
  const int64_t bh = static_cast<int64_t>(b) * p.Hkv + hk;
  for (int c = threadIdx.x; c < kHeadDim; c += kDecodeThreads) is_out[c] = 0;
  __syncthreads();
  if (threadIdx.x < n_out) {
    const int c = min(max(p.idx[bh * n_out + threadIdx.x], 0), kHeadDim - 1);  // stay in bounds on bad input
    idx_s[threadIdx.x] = c;
    is_out[c] = 1;
  }
  __syncthreads();
  const Tq* Qb = static_cast<const Tq*>(p.Q) + (static_cast<int64_t>(b) * p.Hq + hk * G) * kHeadDim;
  for (int e = threadIdx.x; e < G * kHeadDim; e += kDecodeThreads) {
    const int c = e % kHeadDim;
    q_in[e] = is_out[c] ? 0.0f : load_q<Tq>(Qb, e);
  }
  for (int e = threadIdx.x; e < G * n_out; e += kDecodeThreads) {
    const int j = e / n_out, o = e % n_out;
    q_out[j * kMaxOutliers + o] = load_q<Tq>(Qb, j * kHeadDim + idx_s[o]);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += kDecodeThreads) {
    float acc[G];
#pragma unroll
    for (int j = 0; j < G; ++j) acc[j] = 0.0f;
    const uint4* row = reinterpret_cast<const uint4*>(p.S + static_cast<int64_t>(i) * kHeadDim);
#pragma unroll 4
    for (int c8 = 0; c8 < kHeadDim / 8; ++c8) {
      const uint4 w = __ldg(row + c8);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float s0 = __uint_as_float(u[k] << 16), s1 = __uint_as_float(u[k] & 0xFFFF0000u);
        const int c = 8 * c8 + 2 * k;
#pragma unroll
        for (int j = 0; j < G; ++j) {
          acc[j] = fmaf(s0, q_in[j * kHeadDim + c], acc[j]);
          acc[j] = fmaf(s1, q_in[j * kHeadDim + c + 1], acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < G; ++j) sq_in[j * m + i] = acc[j];
  }
  for (int i = threadIdx.x; i < m_out; i += kDecodeThreads) {
    float acc[G];
#pragma unroll
    for (int j = 0; j < G; ++j) acc[j] = 0.0f;
    for (int o = 0; o < n_out; ++o) {
      const float s = __bfloat162float(p.S_out[static_cast<int64_t>(i) * kHeadDim + idx_s[o]]);
#pragma unroll
      for (int j = 0; j < G; ++j) acc[j] = fmaf(s, q_out[j * kMaxOutliers + o], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < G; ++j) sq_out[j * m_out + i] = acc[j];
  }
  __syncthreads();
  for (int pi = warp; pi < 2 * G; pi += kDecodeWarps) {
    const int j = pi >> 1, part = pi & 1;
    const float* v = part ? sq_out + j * m_out : sq_in + j * m;
    const int n = part ? m_out : m;
    float s = 0.0f;
    for (int i = lane; i < n; i += 32) s += v[i];
    s = warp_sum(s);
    if (lane == 0) sums[2 * j + part] = s;
  }
  __syncthreads();

  // ---- scores, online softmax, value accumulation ----
  const float c_in = kSqrtHalfPi / static_cast<float>(m);
  const float c_out = m_out > 0 ? kSqrtHalfPi / static_cast<float>(m_out) : 0.0f;
  const int wpt = m >> 5, wpo = m_out >> 5;
  float run_m[G], run_l[G], acc_o[G][4];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    run_m[j] = -INFINITY;
    run_l[j] = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) acc_o[j][k] = 0.0f;
  }

  for (int tile = t0 + warp * 32; tile < t1; tile += kDecodeThreads) {
    const int t = tile + lane;
    const bool valid = t < t1;
    const int64_t tok = bh * p.cap + (valid ? t : tile);
    float dot_in[G], dot_out[G];
#pragma unroll
    for (int j = 0; j < G; ++j) dot_in[j] = dot_out[j] = 0.0f;
    for (int w = 0; w < wpt; ++w) {
      const uint32_t word = valid ? p.kbits[tok * wpt + w] : 0u;
#pragma unroll 8
      for (int bit = 0; bit < 32; ++bit) {
        if ((word >> bit) & 1u) {
#pragma unroll
          for (int j = 0; j < G; ++j) dot_in[j] += sq_in[j * m + 32 * w + bit];
        }
      }
    }
    for (int w = 0; w < wpo; ++w) {
      const uint32_t word = valid ? p.kbits_out[tok * wpo + w] : 0u;
#pragma unroll 8
      for (int bit = 0; bit < 32; ++bit) {
        if ((word >> bit) & 1u) {
#pragma unroll
          for (int j = 0; j < G; ++j) dot_out[j] += sq_out[j * m_out + 32 * w + bit];
        }
      }
    }
    float nin = 0.0f, nout = 0.0f;
    if (valid) {
      const __half2 nn = reinterpret_cast<const __half2*>(p.knorm)[tok];
      nin = __low2float(nn);
      nout = __high2float(nn);
    }
    float prob[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const float score = c_in * nin * (2.0f * dot_in[j] - sums[2 * j]) +
                          c_out * nout * (2.0f * dot_out[j] - sums[2 * j + 1]);
      if (p.scores != nullptr && valid)
        p.scores[(static_cast<int64_t>(b) * p.Hq + hk * G + j) * p.T + t] = score;
      const float logit = valid ? score * p.sm_scale_log2 : -INFINITY;
      const float new_m = fmaxf(run_m[j], warp_max(logit));  // finite: lane 0 is valid
      const float alpha = exp2f(run_m[j] - new_m);
      prob[j] = valid ? exp2f(logit - new_m) : 0.0f;
      run_l[j] = run_l[j] * alpha + warp_sum(prob[j]);
      run_m[j] = new_m;
#pragma unroll
      for (int k = 0; k < 4; ++k) acc_o[j][k] *= alpha;
    }
    const int n_valid = min(32, t1 - tile);
    const int64_t tok0 = bh * p.cap + tile;
    for (int tt = 0; tt < n_valid; ++tt) {
      const uint32_t codes =
          reinterpret_cast<const uint16_t*>(p.vcode + (tok0 + tt) * (kHeadDim / 2))[lane];
      const uint32_t sz = reinterpret_cast<const uint32_t*>(p.vsz + (tok0 + tt) * (2 * kHeadDim / kValueGroup))[lane >> 3];
      const float scale = __half2float(__ushort_as_half(static_cast<unsigned short>(sz & 0xFFFFu)));
      const float zero = __half2float(__ushort_as_half(static_cast<unsigned short>(sz >> 16)));
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = fmaf(static_cast<float>((codes >> (4 * k)) & 0xFu), scale, zero);
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float pt = __shfl_sync(0xffffffffu, prob[j], tt);
#pragma unroll
        for (int k = 0; k < 4; ++k) acc_o[j][k] = fmaf(pt, v[k], acc_o[j][k]);
      }
    }
  }

  // ---- combine the warps of this CTA ----
#pragma unroll
  for (int j = 0; j < G; ++j) {
#pragma unroll
    for (int k = 0; k < 4; ++k) red[(warp * G + j) * kHeadDim + 4 * lane + k] = acc_o[j][k];
    if (lane == 0) {
      wm[warp * G + j] = run_m[j];
      wl[warp * G + j] = run_l[j];
    }
  }
  __syncthreads();
  const int hq0 = hk * G;
  for (int e = threadIdx.x; e < G * kHeadDim; e += kDecodeThreads) {
    const int j = e / kHeadDim, c = e % kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, wm[w * G + j]);
    float L = 0.0f, ov = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) {
        const float f = exp2f(wm[w * G + j] - M);
        L += wl[w * G + j] * f;
        ov += red[(w * G + j) * kHeadDim + c] * f;
      }
    }
    const int64_t row = static_cast<int64_t>(b) * p.Hq + hq0 + j;
    if (p.splits == 1) {
      p.O[row * kHeadDim + c] = L > 0.0f ? ov / L : 0.0f;
    } else {
      const int64_t prow = row * p.splits + split;
      p.part_o[prow * kHeadDim + c] = ov;
      if (c == 0) {
        p.part_ml[2 * prow] = M;
        p.part_ml[2 * prow + 1] = L;
      }
    }
  }
  if (p.splits == 1) return;

  // ---- last CTA of this (b, hk) merges the splits ----
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.tickets + bh, 1);
    *flag = (prev == p.splits - 1);
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  for (int e = threadIdx.x; e < G * kHeadDim; e += kDecodeThreads) {
    const int j = e / kHeadDim, c = e % kHeadDim;
    const int64_t row = static_cast<int64_t>(b) * p.Hq + hq0 + j;
    float M = -INFINITY;
    for (int s = 0; s < p.splits; ++s) M = fmaxf(M, __ldcg(p.part_ml + 2 * (row * p.splits + s)));
    float L = 0.0f, ov = 0.0f;
    if (M != -INFINITY) {
      for (int s = 0; s < p.splits; ++s) {
        const int64_t prow = row * p.splits + s;
        const float f = exp2f(__ldcg(p.part_ml + 2 * prow) - M);
        L += __ldcg(p.part_ml + 2 * prow + 1) * f;
        ov += __ldcg(p.part_o + prow * kHeadDim + c) * f;
      }
    }
    p.O[row * kHeadDim + c] = L > 0.0f ? ov / L : 0.0f;
  }
  if (threadIdx.x == 0) p.tickets[bh] = 0;  // leave the workspace zeroed for the next call
}

template <int G>
size_t decode_smem_bytes(const DecodeParams& p) {
  return sizeof(float) * (static_cast<size_t>(G) * (p.m + p.m_out + kHeadDim + kMaxOutliers) +
                          static_cast<size_t>(kDecodeWarps) * G * kHeadDim + 2 * kDecodeWarps * G + 2 * G) +
         sizeof(int) * (kMaxOutliers + 1) + kHeadDim;
}

template <int G, typename Tq>
cudaError_t launch_g(const DecodeParams& p, cudaStream_t s) {
  const size_t smem = decode_smem_bytes<G>(p);
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(decode_simt_kernel<G, Tq>), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.splits, p.Hkv, p.B);
  decode_simt_kernel<G, Tq><<<grid, kDecodeThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename Tq>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  switch (p.Hq / p.Hkv) {
    case 1: return launch_g<1, Tq>(p, s);
    case 2: return launch_g<2, Tq>(p, s);
    case 4: return launch_g<4, Tq>(p, s);
    case 8: return launch_g<8, Tq>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, qjl_dtype dt, cudaStream_t s) {
  return dt == QJL_BF16 ? launch_t<__nv_bfloat16>(p, s) : launch_t<float>(p, s);
}

}  // namespace qjl
