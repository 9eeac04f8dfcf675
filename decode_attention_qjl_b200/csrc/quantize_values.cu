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
// Four threads quantise one group of 32 values: each loads 8 consecutive
// values with one 16-byte load (two for fp32), the group's min and max are
// combined with two shuffles, and each thread stores its 8 codes as one
// 32-bit word (4-bit codes) or as two bytes of two 2-bit code lines. Sixteen consecutive threads cover one token's 128 values, so
// loads and stores are contiguous across the warp; every thread does this for
// four tokens, whose loads it issues together.
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

constexpr int kValTokensPerThread = 4;  // tokens per thread: their loads are all in flight together

template <typename Tin, int BITS>
__global__ void __launch_bounds__(256) quantize_values_kernel(ValuesParams p) {
  constexpr int kTop = (1 << BITS) - 1;
  constexpr int kChunks = kHeadDim / 8;  // 16 chunks of 8 values per token
  constexpr int U = kValTokensPerThread;
  // grid (ceil(T / (16 U)), B * Hkv): blockIdx.y is the (b, h) slab; thread i
  // takes chunk i % 16 of tokens 16 (U blockIdx.x + u) + i / 16, u < U
  const int chunk = threadIdx.x % kChunks;
  const int h = blockIdx.y % p.Hkv;
  const int b = blockIdx.y / p.Hkv;
  const int pos0 = p.t_start ? p.t_start[b] : 0;
  float v[U][8];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    // tokens past the end load the last token (whole 16-lane groups, so the
    // shuffles below stay within live data) and store nothing
    const int t = min((blockIdx.x * U + u) * 16 + static_cast<int>(threadIdx.x) / kChunks, p.T - 1);
    load8<Tin>(static_cast<const Tin*>(p.V) + b * p.sb + h * p.sh + t * p.st + chunk * 8, v[u]);
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int t = (blockIdx.x * U + u) * 16 + static_cast<int>(threadIdx.x) / kChunks;
    float lo = v[u][0], hi = v[u][0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
      lo = fminf(lo, v[u][i]);
      hi = fmaxf(hi, v[u][i]);
    }
    // the 4 chunks of a group are 4 consecutive lanes (chunk % 4 == lane % 4 since 16 | 32)
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    const int pos = pos0 + t;
    if (t >= p.T || pos < 0 || pos >= p.cap) continue;
    const __half zero_h = __float2half_rn(lo);
    const __half scale_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), static_cast<float>(kTop)));
    const float zero = __half2float(zero_h);
    const float scale = __half2float(scale_h);
    uint32_t word = 0u;
    if (scale != 0.0f) {
      const float rcp = __frcp_rn(scale);
#pragma unroll
      for (int i = 0; i < 8; i += 2)
        word |= value_code_pair(v[u][i], v[u][i + 1], zero, scale, rcp, kTop, BITS) << (BITS * i);
    }
    int j;
    unsigned char* tile = tile_of(p.tiles, p.tl, static_cast<int64_t>(b) * p.Hkv + h, p.cap, pos, &j);
    if (BITS == 2) {  // dims 8 chunk .. +3 and +4 .. +7: quads 2 (chunk % 4) and +1 of group chunk / 4
      const int g = chunk >> 2, r0 = 2 * (chunk & 3);
      tile[p.tl.vcode + v2_line(g, r0) + j] = static_cast<unsigned char>(word & 0xFFu);
      tile[p.tl.vcode + v2_line(g, r0 + 1) + j] = static_cast<unsigned char>(word >> 8);
    } else {  // 4 words per group; the group's 16 bytes go to its swizzled chunk
      reinterpret_cast<uint32_t*>(tile + p.tl.vcode + j * (kHeadDim / 2))[4 * vcode_chunk(j, chunk >> 2) + (chunk & 3)] =
          word;
    }
    if ((chunk & 3) == 0) {
      const uint32_t sz = static_cast<uint32_t>(__half_as_ushort(scale_h)) |
                          (static_cast<uint32_t>(__half_as_ushort(zero_h)) << 16);
      reinterpret_cast<uint32_t*>(tile + p.tl.vsz + j * (2 * kHeadDim / kValueGroup * 2))[chunk >> 2] = sz;
    }
  }
}

}  // namespace

cudaError_t launch_quantize_values(const ValuesParams& p, qjl_dtype dt, cudaStream_t s) {
  const int threads = 256;  // 16 tokens x 16 chunks per pass, kValTokensPerThread passes
  const int tok_per_block = threads / (kHeadDim / 8) * kValTokensPerThread;
  dim3 grid((p.T + tok_per_block - 1) / tok_per_block, p.B * p.Hkv);
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
