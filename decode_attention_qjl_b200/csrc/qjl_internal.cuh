// Internal declarations shared by the QJL library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "qjl.h"

namespace qjl {

constexpr int kHeadDim = 128;     // d
constexpr int kValueGroup = 32;   // dims per value quantisation group
constexpr int kMaxOutliers = 32;  // n_outlier limit
constexpr int kMaxM = 512;
constexpr int kMaxMOut = 256;
// Decode streams the cache in tiles of this many tokens; the cache capacity
// (tokens per (sequence, kv head) slab) must be a multiple of it so that every
// tile copy stays inside its slab.
constexpr int kDecodeTileTokens = 64;
// Decode streams the cache in stages of up to this many consecutive tiles of
// one (sequence, kv head), one bulk copy each.
constexpr int kStageTiles = 4;

// sqrt(pi/2) in fp32
constexpr float kSqrtHalfPi = 1.2533141373155003f;
constexpr float kLog2e = 1.4426950408889634f;

// 2-bit value codes: one line per (group g, quad r) of dims 32g + 4r .. +3,
// holding the byte of each of the tile's 64 tokens (token j at byte j; the
// lowest dim in the lowest two bits), then 4 bytes of padding, so that the
// lines of the eight quads of a group start in eight different bank pairs.
constexpr int kV2LineBytes = kDecodeTileTokens + 4;
constexpr int kV2Lines = kHeadDim / 4;
__host__ __device__ inline int v2_line(int g, int r) { return (8 * g + r) * kV2LineBytes; }

// Byte offsets of the sections of a 64-token cache tile, and the tile size,
// for 4-bit (vbits = 4) or 2-bit (vbits = 2) value codes.
struct TileLayout {
  int kbits, kbits_out, knorm, vcode, vsz, bytes, vbits;
};
__host__ __device__ inline TileLayout tile_layout(int m, int m_out, int vbits = 4) {
  TileLayout t;
  t.vbits = vbits;
  t.kbits = 0;
  t.kbits_out = t.kbits + kDecodeTileTokens * (m / 8);
  t.knorm = t.kbits_out + kDecodeTileTokens * (m_out / 8);
  t.vcode = t.knorm + kDecodeTileTokens * 4;
  t.vsz = t.vcode + (vbits == 2 ? kV2Lines * kV2LineBytes : kDecodeTileTokens * (kHeadDim / 2));
  t.bytes = t.vsz + kDecodeTileTokens * (kHeadDim / 32) * 4;
  return t;
}
// Value codes of token j of a tile: the 16 bytes of group g (dims 32g .. 32g+31)
// sit at 16-byte chunk g ^ ((j >> 1) & 3) of the token's 64 bytes, so that eight
// consecutive tokens' chunks of one group fall in eight different shared-memory
// bank quads when a tile is staged.
__host__ __device__ inline int vcode_chunk(int j, int g) { return g ^ ((j >> 1) & 3); }
// Start of the tile that holds token slot `pos` of slab `bh`, and the slot within it.
__host__ __device__ inline unsigned char* tile_of(unsigned char* tiles, const TileLayout& tl, int64_t bh, int cap,
                                                  int pos, int* j) {
  *j = pos % kDecodeTileTokens;
  return tiles + (bh * (cap / kDecodeTileTokens) + pos / kDecodeTileTokens) * static_cast<int64_t>(tl.bytes);
}

// 4-bit value code of v in a group with fp16 zero point `zero` and step
// `scale` (both as fp32, scale > 0), `rcp` = fp32(1 / scale): the code that
// clamp(rint(fp32(fp32(v - zero) / scale)), 0, 15) gives with every step an
// IEEE fp32 operation rounded to nearest even, without a division per value.
// y = t * rcp is within 2^-19 of x = t / scale (|x| < 17: two roundings of
// relative size 2^-24 each), so away from the half-way points k + 1/2 the
// code is rint(y). Within 2^-17 of one, the fp32 quotient itself is taken:
// the fp64 quotient rounded to fp32, which equals the correctly rounded fp32
// quotient because a 53-bit intermediate makes double rounding of a 24-bit
// division innocuous (S. A. Figueroa, "When is double rounding innocuous?",
// SIGNUM Newsletter 30(3), 1995).
// Rounding is done on the FMA pipe: for |y| < 2^22, fp32(y + 1.5 * 2^23) has
// an ulp of 1, so the addition itself rounds y to the nearest integer (ties
// to even) and the integer is the sum's low mantissa bits; subtracting
// 1.5 * 2^23 again gives rint(y) exactly (the callers keep y in [0, 15]).
__device__ __forceinline__ int value_rint(float y, float* r) {
  const float s = __fadd_rn(y, 12582912.0f);  // 1.5 * 2^23
  *r = __fsub_rn(s, 12582912.0f);
  return __float_as_int(s) - 0x4B400000;      // the bits of 1.5 * 2^23
}
// The code for 2^bits - 1 = `top` levels above zero (the same steps; 15 for
// the cache's 4-bit values). y is clamped to [0, top] before rounding:
// rint(clamp(y)) = clamp(rint(y)) for these bounds, and a value whose
// quotient lies outside the levels takes the end code either way.
__device__ __forceinline__ uint32_t value_code(float v, float zero, float scale, float rcp, int top = 15) {
  const float t = __fsub_rn(v, zero);
  const float y = fminf(fmaxf(__fmul_rn(t, rcp), 0.0f), static_cast<float>(top));
  float r;
  int k = value_rint(y, &r);
  if (fabsf(__fsub_rn(y, r)) >= 0.5f - 7.62939453125e-6f) {  // within 2^-17 of a half-way point
    const float x = __double2float_rn(__ddiv_rn(static_cast<double>(t), static_cast<double>(scale)));
    k = value_rint(fminf(fmaxf(x, 0.0f), static_cast<float>(top)), &r);
  }
  return static_cast<uint32_t>(k);
}

// Two values' codes at once (low code in bits 0.., the second `bits` higher),
// the same steps with the element-wise pair instructions of sm_100 (each
// element an IEEE fp32 operation rounded to nearest even, as above).
__device__ __forceinline__ unsigned long long f32x2_pack(float a, float b) {
  return static_cast<unsigned long long>(__float_as_uint(a)) |
         (static_cast<unsigned long long>(__float_as_uint(b)) << 32);
}
__device__ __forceinline__ float f32x2_lo(unsigned long long x) { return __uint_as_float(static_cast<uint32_t>(x)); }
__device__ __forceinline__ float f32x2_hi(unsigned long long x) {
  return __uint_as_float(static_cast<uint32_t>(x >> 32));
}
__device__ __forceinline__ uint32_t value_code_pair(float v0, float v1, float zero, float scale, float rcp, int top,
                                                    int bits) {
  unsigned long long t, y, sm, r, d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(f32x2_pack(v0, v1)), "l"(f32x2_pack(zero, zero)));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(t), "l"(f32x2_pack(rcp, rcp)));
  const float ftop = static_cast<float>(top);
  const float y0 = fminf(fmaxf(f32x2_lo(y), 0.0f), ftop), y1 = fminf(fmaxf(f32x2_hi(y), 0.0f), ftop);
  const unsigned long long yc = f32x2_pack(y0, y1), magic = f32x2_pack(12582912.0f, 12582912.0f);  // 1.5 * 2^23
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(sm) : "l"(yc), "l"(magic));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(sm), "l"(magic));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(yc), "l"(r));
  int k0 = static_cast<int>(static_cast<uint32_t>(sm)) - 0x4B400000;
  int k1 = static_cast<int>(static_cast<uint32_t>(sm >> 32)) - 0x4B400000;
  constexpr float kNear = 0.5f - 7.62939453125e-6f;  // within 2^-17 of a half-way point
  if (fabsf(f32x2_lo(d)) >= kNear) {
    const float x = __double2float_rn(__ddiv_rn(static_cast<double>(f32x2_lo(t)), static_cast<double>(scale)));
    float rr;
    k0 = value_rint(fminf(fmaxf(x, 0.0f), ftop), &rr);
  }
  if (fabsf(f32x2_hi(d)) >= kNear) {
    const float x = __double2float_rn(__ddiv_rn(static_cast<double>(f32x2_hi(t)), static_cast<double>(scale)));
    float rr;
    k1 = value_rint(fminf(fmaxf(x, 0.0f), ftop), &rr);
  }
  return static_cast<uint32_t>(k0) | (static_cast<uint32_t>(k1) << bits);
}

// Eight values' codes (value i in bits bits * i ..): the steps of
// value_code_pair on four pairs, with one test of the distance to the
// half-way points for all eight (values near one take the exact quotient, one
// by one, as there).
__device__ __forceinline__ uint32_t value_codes8(const float (&v)[8], float zero, float scale, float rcp, int top,
                                                 int bits) {
  const float ftop = static_cast<float>(top);
  const unsigned long long zz = f32x2_pack(zero, zero), rr = f32x2_pack(rcp, rcp);
  const unsigned long long magic = f32x2_pack(12582912.0f, 12582912.0f);  // 1.5 * 2^23
  constexpr float kNear = 0.5f - 7.62939453125e-6f;                      // within 2^-17 of a half-way point
  uint32_t word = 0u;
  float dmax = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    unsigned long long t, y, sm, r, d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(t) : "l"(f32x2_pack(v[2 * k], v[2 * k + 1])), "l"(zz));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(t), "l"(rr));
    const float y0 = fminf(fmaxf(f32x2_lo(y), 0.0f), ftop), y1 = fminf(fmaxf(f32x2_hi(y), 0.0f), ftop);
    const unsigned long long yc = f32x2_pack(y0, y1);
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(sm) : "l"(yc), "l"(magic));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(sm), "l"(magic));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(yc), "l"(r));
    const uint32_t k0 = static_cast<uint32_t>(sm) - 0x4B400000u, k1 = static_cast<uint32_t>(sm >> 32) - 0x4B400000u;
    word |= (k0 | (k1 << bits)) << (2 * bits * k);
    dmax = fmaxf(dmax, fmaxf(fabsf(f32x2_lo(d)), fabsf(f32x2_hi(d))));
  }
  if (dmax >= kNear) {
    const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // unrolled: v stays in registers
      const float t = __fsub_rn(v[i], zero);
      const float y = fminf(fmaxf(__fmul_rn(t, rcp), 0.0f), ftop);
      float r;
      value_rint(y, &r);
      if (fabsf(__fsub_rn(y, r)) >= kNear) {
        const float x = __double2float_rn(__ddiv_rn(static_cast<double>(t), static_cast<double>(scale)));
        const uint32_t k = static_cast<uint32_t>(value_rint(fminf(fmaxf(x, 0.0f), ftop), &r));
        word = (word & ~(mask << (bits * i))) | (k << (bits * i));
      }
    }
  }
  return word;
}

struct KeysParams {
  const void* K;
  int64_t sb, sh, st;  // element strides
  int B, Hkv, T, cap;
  const int32_t* t_start;
  int m, m_out, n_out;
  const __nv_bfloat16* S;      // [m, d]
  const __nv_bfloat16* St;     // [d, m] (S transposed)
  const __nv_bfloat16* S_out;  // [m_out, d]
  int32_t* idx;                // [B, Hkv, n_out]
  unsigned char* tiles;        // cache tiles (layout in qjl.h)
  TileLayout tl;
  double* energy;              // workspace [B, Hkv, d] (prefill)
  float guard;                 // relative guard band of the fp32 sign decision (CUDA-core sketch)
  float guard_tc;              // the same for the tensor-core sketch (no 2^-10 floor)
  const void* S_img;           // S then S_out in the tcgen05 B-operand layout (quantize_keys_tc.cu)
  int num_sms;
};

struct ValuesParams {
  const void* V;
  int64_t sb, sh, st;
  int B, Hkv, T, cap;
  const int32_t* t_start;
  unsigned char* tiles;  // cache tiles (layout in qjl.h; tl.vbits: 4- or 2-bit codes)
  TileLayout tl;
};

struct DecodeParams {
  const void* Q;      // [B, Hq, d]
  const void* K_new;  // decode step: the appended token's key, element (b, h, c) at b * k_sb + h * k_sh + c
  const void* V_new;  // decode step: the appended token's value, likewise with v_sb, v_sh
  int64_t k_sb, k_sh, v_sb, v_sh;
  int append;         // 1: a decode step (append one token per sequence, then attend over it too)
  int B, Hq, Hkv, T, cap;
  const int32_t* seqlens;
  int m, m_out, n_out;
  const __nv_bfloat16* S;      // [m, d]
  const __nv_bfloat16* S_out;  // [m_out, d]
  // S then S_out in the A-fragment order of a bf16 m16n8k16 MMA: 16-row tile mt,
  // 16-channel step ks, lane l -> S_frag[(mt * 8 + ks) * 32 + l] (see decode_fill_s_frag)
  const uint4* S_frag;
  float guard;        // relative guard band of the appended key's sign decision (tensor-core sums)
  const int32_t* idx;
  unsigned char* tiles;  // cache tiles (layout in qjl.h); a decode step writes the appended token
  TileLayout tl;
  float sm_scale_log2;  // sm_scale * log2(e)
  float* O;             // [B, Hq, d]
  float* ML;            // [B, Hq, 2] or null: O is then the unnormalised part, ML its (max, sum) in log2 units
  float* scores;        // [B, Hq, score_stride] or null
  int score_stride;
  int grid;             // CTAs (at most one per SM)
  int nstage;           // cache stages of kStageTiles tiles in the shared-memory ring
  int* hdr;             // workspace header: [2] error bits (the rest is reserved, zero)
  int* tickets;         // [B * Hkv] merge counters, zero at rest
  unsigned char* qblock;  // [B * Hkv][qblock_bytes] query blocks of segments past a CTA's first two
  int qblock_bytes;
  float* part_o;        // [2 * grid][G][d] partial outputs of the pairs shared by several CTAs
  float* part_ml;       // [2 * grid][G][2] their running maxima and sums
  int q_fp32;           // Q (and K_new, V_new) are fp32 (else bf16)
  unsigned long long wait_cycles;  // limit of every wait inside the kernel, in SM clock cycles
};

constexpr int kDecodeQBuffers = 2;  // query-block buffers per CTA in shared memory
// Error bits of the decode workspace header (hdr[2]).
constexpr int kDecodeErrTimeout = 1;

// Bytes of the prepared query sketch that decode builds per (sequence, kv head):
// per-lane score-MMA B fragments, then the fixed-point exponents (int32 [G][2])
// and sums (int64 [G][2]); a multiple of 16 bytes.
__host__ __device__ inline size_t decode_qblock_bytes(int G, int m, int m_out) {
  const int nts = (G + 1) / 2;  // score MMA N-tiles: 8 columns = 2 heads x 4 limbs
  const size_t frag = static_cast<size_t>(nts) * (m / 32 + m_out / 32) * 2 * 32 * 4;
  return (frag + 24 * static_cast<size_t>(G) + 15) & ~static_cast<size_t>(15);
}

// Decode workspace layout: a 256-byte header, the merge counters, a query
// block slot per (sequence, kv head) (used by the pairs that are not among a
// CTA's first two segments) and the partial results of the pairs whose tiles
// are split between CTAs (two slots per CTA: its first and its last pair).
// The header and the counters must be zero before a call; every call leaves
// the counters at zero.
struct DecodeWsLayout {
  size_t hdr, tickets, qblock, part_o, part_ml, zero_bytes, total;
};
inline DecodeWsLayout decode_ws_layout(int B, int Hq, int Hkv, int num_sms, int m, int m_out) {
  auto a256 = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  DecodeWsLayout w{};
  const size_t bh = static_cast<size_t>(B) * Hkv;
  const int G = Hq / Hkv;
  w.hdr = 0;
  w.tickets = 256;
  w.qblock = w.tickets + a256(bh * sizeof(int));
  w.zero_bytes = w.qblock;
  w.part_o = w.qblock + a256(bh * decode_qblock_bytes(G, m, m_out));
  w.part_ml = w.part_o + a256(static_cast<size_t>(2) * num_sms * G * kHeadDim * sizeof(float));
  w.total = w.part_ml + a256(static_cast<size_t>(2) * num_sms * G * 2 * sizeof(float));
  return w;
}

// Launchers (return the cudaGetLastError() of the launches).
cudaError_t launch_quantize_values(const ValuesParams& p, qjl_dtype dt, cudaStream_t s);
int64_t exact_decode_chunks(int cap);
cudaError_t launch_exact_decode(int fmt, const void* K, const void* V, float k_scale, float v_scale, int B, int Hq,
                                int Hkv, int cap, int T, const void* Q, int q_fp32, const int32_t* seqlens,
                                float sm_scale_log2, float* O, float* ws, cudaStream_t s);
cudaError_t launch_fp8_quantize(const void* x, int q_fp32, int64_t n, float scale, unsigned char* out, cudaStream_t s);
cudaError_t launch_minmax_quantize(const void* x, int q_fp32, int64_t n_rows, int bits, unsigned char* out,
                                   cudaStream_t s);
int exact_row_bytes(int fmt);  // bytes of one cached token of one kv head (K or V) in a comparison format
cudaError_t launch_merge_partials(const float* O_parts, int64_t o_stride, const float* ML_parts, int64_t ml_stride,
                                  int R, int64_t rows, float* O, cudaStream_t s);
cudaError_t launch_channel_energy(const KeysParams& p, qjl_dtype dt, cudaStream_t s);
cudaError_t launch_select_outliers(const KeysParams& p, cudaStream_t s);
cudaError_t launch_sketch_keys(const KeysParams& p, qjl_dtype dt, cudaStream_t s);
// tensor-core sign sketch (quantize_keys_tc.cu)
bool sketch_keys_tc_applies(const KeysParams& p, qjl_dtype dt);
cudaError_t launch_sketch_keys_tc(const KeysParams& p, int num_sms, cudaStream_t s);
void tc_fill_s_image(const uint16_t* S, int rows, uint16_t* img);  // host: [rows, d] -> image [rows * d]
cudaError_t launch_decode(const DecodeParams& p, qjl_dtype dt, cudaStream_t s);
// host: S [m, d] and S_out [m_out, d] (bf16 bits) -> S_frag [(m + m_out) * d] (decode.cu)
void decode_fill_s_frag(const uint16_t* S, const uint16_t* S_out, int m, int m_out, uint16_t* out);

// Bytes at the start of a decode workspace that must be zero before a call
// (header and merge counters); 0 for an invalid shape.
size_t decode_ws_zero_bytes(const qjl_ctx* ctx, int B, int Hq, int Hkv);
// The device a context was created on (-1 for null).
int ctx_device(const qjl_ctx* ctx);

// Raise a kernel's dynamic shared-memory limit to at least `bytes`. The
// attribute is set only when the limit grows, so steady-state calls enqueue
// nothing but the launch (and stay legal inside CUDA stream capture).
cudaError_t ensure_smem_limit(const void* func, size_t bytes);

// Record the message that qjl_last_error() returns on this thread.
void set_last_error(const std::string& msg);

// Host-side sketch generation (bf16 bit patterns).
void sketch_fill_host(uint64_t seed, uint64_t counter_offset, int rows, int d, uint16_t* out);
constexpr uint64_t kSketchOutOffset = 1ull << 62;

}  // namespace qjl
