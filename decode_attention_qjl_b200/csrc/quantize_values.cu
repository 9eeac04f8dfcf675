// Token-wise asymmetric 4-bit value quantisation, groups of 32 dims.
//
// QJL summary (atlas.scime.ai), Limitations: values use standard token-wise
// quantisation. The grid is the min-max one of "2 numbers out of 128 destroy
// the entire KV cache" (Towards AI), section "The Obvious Fix: Use Fewer
// Bits": zero = min, 16 equally spaced levels up to max, nearest level.
// zero and scale are stored as fp16; every arithmetic step is one IEEE fp32
// operation with round-to-nearest-even, so the code decision is reproducible.
//
// One thread quantises one group of 32 values (64 B of bf16 or 128 B of fp32,
// loaded as 16-byte vectors) and writes 16 B of codes plus 4 B of scale/zero.
// Consecutive threads own consecutive groups, so the stores are contiguous.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

template <typename Tin>
__device__ __forceinline__ void load_group(const Tin* src, float (&v)[32]);

template <>
__device__ __forceinline__ void load_group<__nv_bfloat16>(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 w = __ldg(s4 + j);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * j + 2 * k] = __uint_as_float(u[k] << 16);
      v[8 * j + 2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
    }
  }
}

template <>
__device__ __forceinline__ void load_group<float>(const float* src, float (&v)[32]) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 w = __ldg(s4 + j);
    v[4 * j] = w.x;
    v[4 * j + 1] = w.y;
    v[4 * j + 2] = w.z;
    v[4 * j + 3] = w.w;
  }
}

template <typename Tin>
__global__ void __launch_bounds__(256) quantize_values_kernel(ValuesParams p) {
  constexpr int kGroups = kHeadDim / kValueGroup;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(p.B) * p.Hkv * p.T * kGroups;
  if (gid >= total) return;
  const int g = static_cast<int>(gid % kGroups);
  int64_t r = gid / kGroups;
  const int t = static_cast<int>(r % p.T);
  r /= p.T;
  const int h = static_cast<int>(r % p.Hkv);
  const int b = static_cast<int>(r / p.Hkv);
  const int pos = (p.t_start ? p.t_start[b] : 0) + t;
  if (pos < 0 || pos >= p.cap) return;

  const Tin* src = static_cast<const Tin*>(p.V) + b * p.sb + h * p.sh + t * p.st + g * kValueGroup;
  float v[32];
  load_group<Tin>(src, v);

  float lo = v[0], hi = v[0];
#pragma unroll
  for (int i = 1; i < 32; ++i) {
    lo = fminf(lo, v[i]);
    hi = fmaxf(hi, v[i]);
  }
  const __half zero_h = __float2half_rn(lo);
  const __half scale_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
  const float zero = __half2float(zero_h);
  const float scale = __half2float(scale_h);

  uint32_t words[4] = {0u, 0u, 0u, 0u};
  if (scale != 0.0f) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float c = rintf(__fdiv_rn(__fsub_rn(v[i], zero), scale));
      c = fminf(fmaxf(c, 0.0f), 15.0f);
      words[i >> 3] |= static_cast<uint32_t>(c) << (4 * (i & 7));
    }
  }
  const int64_t tok = (static_cast<int64_t>(b) * p.Hkv + h) * p.cap + pos;
  reinterpret_cast<uint4*>(p.vcode + tok * (kHeadDim / 2))[g] = make_uint4(words[0], words[1], words[2], words[3]);
  const uint32_t sz = static_cast<uint32_t>(__half_as_ushort(scale_h)) |
                      (static_cast<uint32_t>(__half_as_ushort(zero_h)) << 16);
  reinterpret_cast<uint32_t*>(p.vsz + tok * (2 * kGroups))[g] = sz;
}

}  // namespace

cudaError_t launch_quantize_values(const ValuesParams& p, qjl_dtype dt, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(p.B) * p.Hkv * p.T * (kHeadDim / kValueGroup);
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (dt == QJL_BF16)
    quantize_values_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  else
    quantize_values_kernel<float><<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace qjl
