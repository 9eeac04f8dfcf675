// Token-wise asymmetric 4-bit (or 2-bit) value quantisation, groups of 32 dims.
//
// QJL summary (atlas.scime.ai), Limitations: values use standard token-wise
// quantisation. The grid is the min-max one of "2 numbers out of 128 destroy
// the entire KV cache" (Towards AI), section "The Obvious Fix: Use Fewer
// Bits": zero = min, 16 (or 4) equally spaced levels up to max, nearest level.
// zero and scale are stored as fp16; the code is the one that every step as
// one IEEE fp32 operation with round-to-nearest-even gives (value_code: a
// reciprocal multiply, with the exact fp32 quotient near the half-way points),
// so the code decision is reproducible.
//
// One thread quantises one group of 32 values of one token: four 16-byte
// loads (eight for fp32), the min and max in registers, the scale and zero
// once, and the 16 code bytes with one 16-byte store (4-bit codes) or eight
// bytes into the group's 2-bit code lines. Four consecutive threads cover one
// token's 128 values, so loads and stores are contiguous across the warp.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

template <typename Tin>
__device__ __forceinline__ void load8(const Tin* src, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(u[k] << 16);
    v[2 * k + 1] = __uint_as_float(u[k] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void load8<float>(const float* src, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int kValThreads = 256;                            // 64 tokens x 4 groups per block
constexpr int kValGroups = kHeadDim / kValueGroup;         // 4 groups per token
constexpr int kValTokensPerBlock = kValThreads / kValGroups;

template <typename Tin, int BITS>
__global__ void __launch_bounds__(kValThreads, 4) quantize_values_kernel(ValuesParams p) {
  constexpr int kTop = (1 << BITS) - 1;
  // grid (ceil(T / 64), B * Hkv): blockIdx.y is the (b, h) slab; thread i
  // takes group i % 4 of token 64 blockIdx.x + i / 4
  const int g = threadIdx.x % kValGroups;
  const int h = blockIdx.y % p.Hkv;
  const int b = blockIdx.y / p.Hkv;
  const int t = blockIdx.x * kValTokensPerBlock + static_cast<int>(threadIdx.x) / kValGroups;
  const int pos = (p.t_start ? p.t_start[b] : 0) + t;
  if (t >= p.T || pos < 0 || pos >= p.cap) return;
  const Tin* src = static_cast<const Tin*>(p.V) + b * p.sb + h * p.sh + t * p.st + g * kValueGroup;
  float v[4][8];
#pragma unroll
  for (int c = 0; c < 4; ++c) load8<Tin>(src + 8 * c, v[c]);
  float lo = v[0][0], hi = v[0][0];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo = fminf(lo, v[c][i]);
      hi = fmaxf(hi, v[c][i]);
    }
  const __half zero_h = __float2half_rn(lo);
  const __half scale_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), static_cast<float>(kTop)));
  const float zero = __half2float(zero_h);
  const float scale = __half2float(scale_h);
  uint32_t word[4] = {0u, 0u, 0u, 0u};  // dims 8c .. 8c + 7 of the group in word c
  if (scale != 0.0f) {
    const float rcp = __frcp_rn(scale);
#pragma unroll
    for (int c = 0; c < 4; ++c) word[c] = value_codes8(v[c], zero, scale, rcp, kTop, BITS);
  }
  int j;
  unsigned char* tile = tile_of(p.tiles, p.tl, static_cast<int64_t>(b) * p.Hkv + h, p.cap, pos, &j);
  if (BITS == 2) {  // dims 8c .. 8c + 3 and + 4 .. + 7: lines 2c and 2c + 1 of the group
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tile[p.tl.vcode + v2_line(g, 2 * c) + j] = static_cast<unsigned char>(word[c] & 0xFFu);
      tile[p.tl.vcode + v2_line(g, 2 * c + 1) + j] = static_cast<unsigned char>(word[c] >> 8);
    }
  } else {  // the group's 16 bytes go to its swizzled chunk
    *reinterpret_cast<uint4*>(tile + p.tl.vcode + j * (kHeadDim / 2) + 16 * vcode_chunk(j, g)) =
        make_uint4(word[0], word[1], word[2], word[3]);
  }
  const uint32_t sz = static_cast<uint32_t>(__half_as_ushort(scale_h)) |
                      (static_cast<uint32_t>(__half_as_ushort(zero_h)) << 16);
  reinterpret_cast<uint32_t*>(tile + p.tl.vsz + j * (2 * kHeadDim / kValueGroup * 2))[g] = sz;
}

}  // namespace

cudaError_t launch_quantize_values(const ValuesParams& p, qjl_dtype dt, cudaStream_t s) {
  const int threads = kValThreads;
  dim3 grid((p.T + kValTokensPerBlock - 1) / kValTokensPerBlock, p.B * p.Hkv);
  if (p.tl.vbits == 2) {
    if (dt == QJL_BF16)
      quantize_values_kernel<__nv_bfloat16, 2><<<grid, threads, 0, s>>>(p);
    else
      quantize_values_kernel<float, 2><<<grid, threads, 0, s>>>(p);
  } else {
    if (dt == QJL_BF16)
      quantize_values_kernel<__nv_bfloat16, 4><<<grid, threads, 0, s>>>(p);
    else
      quantize_values_kernel<float, 4><<<grid, threads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace qjl
