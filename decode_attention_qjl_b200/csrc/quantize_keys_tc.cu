// QJL key sign sketch on the tensor cores (tcgen05), for bf16 keys in bulk.
//
// QJL summary (atlas.scime.ai), Approach: the key is multiplied by the random
// Gaussian JL matrix S and only sign(S k_in) is kept, plus the norm; the
// outlier channels get their own sketch sign(S_out k_out) and norm. For a
// block of 128 tokens of one (sequence, kv head) the inlier projection is the
// dense product P = K_in S^T (128 x d times d x m), which this kernel runs as
// tcgen05.mma (bf16 x bf16, fp32 accumulation in tensor memory):
//   * S is kept in shared memory for the whole kernel: qjl_init stores it in
//     global memory already in the 128-byte-swizzled K-major layout of a
//     tcgen05 B operand, so one cp.async.bulk brings it in;
//   * thread r of the CTA loads token r's key row (256 bytes), zeroes its
//     outlier channels, writes it in the same swizzled layout as the A operand
//     and sums the squared norm (compensated fp32, exact to ~2^-48);
//   * one thread issues the d/16 MMAs (K = 16 each) and commits them to an
//     mbarrier; meanwhile every thread computes its token's outlier sketch
//     (n_out exact products per row, fp32 sum with an error bound, fp64 when
//     the bound does not settle the sign);
//   * each warp reads its 32 accumulator rows from tensor memory with
//     tcgen05.ld (thread r receives token r's projections, 32 columns per
//     load), so one thread packs a whole sign word without a ballot.
// A projection whose magnitude is below twice the context's guard band times
// |k_in| is recomputed in fp64 (exact bf16 products, from the operands in
// shared memory, by the whole warp) before its sign is taken, so the bits
// equal the signs of the exact projections, as in the CUDA-core path. Work
// items (b, kv head, 128-token block) are walked by persistent CTAs; the
// tensor-memory columns a CTA allocates times the CTAs that fit on an SM never
// exceed the 512 columns of an SM, so the allocation cannot block.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

constexpr int kTcRows = 128;                // tokens per MMA block (M)
constexpr int kTcThreads = 256;             // two threads per token row (one per 64-channel half)
constexpr int kTcARegion = kTcRows * 128;   // bytes of one 64-channel half of the A block
constexpr uint64_t kTcWaitNs = 2000000000ull;
constexpr int kTcMaxOut = 8;                // outlier channels this kernel handles (more: the CUDA-core path)

__device__ __forceinline__ uint32_t tc_smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t tc_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool tc_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(tc_smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __noinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
  if (tc_try_wait(bar, parity)) return true;
  const uint64_t t0 = tc_timer();
  while (!tc_try_wait(bar, parity))
    if (tc_timer() - t0 > kTcWaitNs) return false;
  return true;
}

// 32 consecutive fp32 accumulator columns of this warp's 32 tensor-memory lanes
// (thread i receives lane i), without the wait.
__device__ __forceinline__ void tc_ld32(uint32_t (&v)[32], uint32_t taddr) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzle layout: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address
  d |= static_cast<uint64_t>(1) << 16;                           // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;                   // stride byte offset: next 8 rows
  d |= static_cast<uint64_t>(1) << 46;                           // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                           // 128-byte swizzle
  return d;
}
// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major, M = 128.
__host__ __device__ constexpr uint32_t tc_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | ((kTcRows >> 4) << 24);
}

// tensor-memory columns for m accumulator columns (a power of two, at least 32)
__host__ __device__ inline int tc_tmem_cols(int m) {
  int c = 32;
  while (c < m) c <<= 1;
  return c;
}

// fp16 bits of sqrt(S) from an fp32 sum of squares s with |s - S| <= rel S:
// sqrt(s) is within rel / 2 + 2^-24 of sqrt(S), and both ends of that interval
// (widened by the rounding of the two products) must round to the same fp16
// value; else -1 (the caller recomputes the norm exactly).
__device__ __forceinline__ int tc_norm_fp16(float s, float rel) {
  const float n = sqrtf(s);
  const float e = 0.5f * rel + 4.0f * 0x1p-24f;
  const unsigned short lo = __half_as_ushort(__float2half_rn(n * (1.0f - e)));
  const unsigned short hi = __half_as_ushort(__float2half_rn(n * (1.0f + e)));
  return lo == hi ? static_cast<int>(lo) : -1;
}

struct TcSmem {
  int a, b, so, nrm, misc, total;
  __host__ __device__ TcSmem(int m, int m_out, int n_out) {
    a = 0;                                         // A block: 2 halves of kTcARegion
    b = a + 2 * kTcARegion;                        // S image: m rows x 256 bytes
    so = b + m * kHeadDim * 2;                     // float [m_out][kTcMaxOut] (0 past n_out)
    nrm = so + m_out * kTcMaxOut * 4;              // float [2 halves][128 rows]: partial |k_in|^2
    misc = nrm + 2 * kTcRows * 4;                  // idx [32], outlier mask [4 words], mbarriers, tmem address
    total = misc + kMaxOutliers * 4 + 16 + 32 + 16 + 16;  // ... + max row norm of S_out at the outlier channels
  }
};

// 256 threads: warp w handles token rows 32 (w mod 4) .. +31 (the tensor-memory
// lanes a warp may read) and channel half w / 4 of them.
__global__ void __launch_bounds__(kTcThreads, 2) sketch_keys_tc_kernel(KeysParams p, int n_items, int tiles_per_bh) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // the swizzle of the MMA operands is a function of address bits 7..9: the
  // operand regions start on 1024-byte boundaries (1 KB is requested extra)
  unsigned char* smem = smem_raw + ((1024u - (tc_smem_u32(smem_raw) & 1023u)) & 1023u);
  const int m = p.m, m_out = p.m_out, n_out = p.n_out;
  const int wpt = m >> 5, wpo = m_out >> 5;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, hf = warp >> 2;
  const int r = 32 * quarter + lane;  // token row of this thread
  const TcSmem L(m, m_out, n_out);
  float* So = reinterpret_cast<float*>(smem + L.so);
  float* nrm_s = reinterpret_cast<float*>(smem + L.nrm);
  int* idx_s = reinterpret_cast<int*>(smem + L.misc);
  uint32_t* omask = reinterpret_cast<uint32_t*>(idx_s + kMaxOutliers);  // 128-bit outlier channel mask
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(omask + 4);            // S image loaded
  uint64_t* bar_mma = bar_s + 1;                                        // MMAs of the current block done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 1);
  unsigned int* so_max_bits = tmem_slot + 4;  // max_i |S_out[i, idx]| (fp32 bits; non-negative)
  const int tcols = tc_tmem_cols(m);

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem_u32(bar_s)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tc_smem_u32(bar_mma)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem_u32(tmem_slot)),
                 "r"(tcols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {  // the swizzled S image, once per CTA
    const uint32_t bytes = static_cast<uint32_t>(m) * kHeadDim * 2;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_smem_u32(bar_s)), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            tc_smem_u32(smem + L.b)),
        "l"(p.S_img), "r"(bytes), "r"(tc_smem_u32(bar_s))
        : "memory");
  }
  const float thr_rel = 2.0f * p.guard;
  const uint32_t a_base = tc_smem_u32(smem + L.a), b_base = tc_smem_u32(smem + L.b);

  // this thread's half row of a block's key: issued one block ahead
  auto key_half = [&](int item, uint4 (&w)[8]) {
    const int64_t bh = item / tiles_per_bh;
    const int b = static_cast<int>(bh / p.Hkv), h = static_cast<int>(bh % p.Hkv);
    const int t = (item % tiles_per_bh) * kTcRows + r;
    const int pos = (p.t_start ? p.t_start[b] : 0) + t;
    const bool live = t < p.T && pos >= 0 && pos < p.cap;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.K) + b * p.sb + h * p.sh +
                                                     static_cast<int64_t>(t) * p.st + 64 * hf);
#pragma unroll
    for (int c = 0; c < 8; ++c) w[c] = live ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 kh[8];
  // this CTA's blocks are a contiguous range, so that consecutive blocks
  // mostly share their (b, kv head) and its outlier channels
  const int per = n_items / gridDim.x, extra = n_items % gridDim.x;
  const int item_begin = blockIdx.x * per + min(static_cast<int>(blockIdx.x), extra);
  const int item_end = item_begin + per + (static_cast<int>(blockIdx.x) < extra ? 1 : 0);
  if (item_begin < item_end) key_half(item_begin, kh);
  bool ok = __syncthreads_and(tc_wait(bar_s, 0)) != 0;

  int64_t cur_bh = -1;
  int local = 0;
  for (int item = item_begin; item < item_end && ok; ++item, ++local) {
    const int64_t bh = item / tiles_per_bh;
    const int tile = item % tiles_per_bh;
    const int b = static_cast<int>(bh / p.Hkv), h = static_cast<int>(bh % p.Hkv);
    if (bh != cur_bh) {  // outlier channels and the S_out columns at them
      if (tid < 4) omask[tid] = 0u;
      if (tid == 0) *so_max_bits = 0u;
      __syncthreads();
      if (tid < n_out) {
        const int c = min(max(p.idx[bh * n_out + tid], 0), kHeadDim - 1);  // stay in bounds on bad input
        idx_s[tid] = c;
        atomicOr(&omask[c >> 5], 1u << (c & 31));
      }
      __syncthreads();
      for (int i = tid; i < m_out; i += kTcThreads) {
        float row[kTcMaxOut];
        float n2 = 0.0f;
#pragma unroll
        for (int o = 0; o < kTcMaxOut; ++o) {
          row[o] = o < n_out ? __bfloat162float(p.S_out[static_cast<int64_t>(i) * kHeadDim + idx_s[o]]) : 0.0f;
          n2 = fmaf(row[o], row[o], n2);
        }
        float4* dst = reinterpret_cast<float4*>(So + i * kTcMaxOut);
        dst[0] = make_float4(row[0], row[1], row[2], row[3]);
        dst[1] = make_float4(row[4], row[5], row[6], row[7]);
        atomicMax(so_max_bits, __float_as_uint(sqrtf(n2) * 1.001f));  // rounded up a little
      }
      cur_bh = bh;
    }
    const int t = tile * kTcRows + r;
    const int pos = (p.t_start ? p.t_start[b] : 0) + t;
    const bool live = t < p.T && pos >= 0 && pos < p.cap;
    const __nv_bfloat16* krow = static_cast<const __nv_bfloat16*>(p.K) + b * p.sb + h * p.sh +
                                static_cast<int64_t>(t) * p.st;
    // ---- half row into the A block (outlier channels zeroed); its squared norm
    const uint32_t om = omask[2 * hf] | 0u, om2 = omask[2 * hf + 1];
    float ss0 = 0.0f, ss1 = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {  // channels 64hf + 8c .. +7
      uint32_t u[4] = {kh[c].x, kh[c].y, kh[c].z, kh[c].w};
      const uint32_t bits = ((c < 4 ? om : om2) >> ((c & 3) * 8)) & 0xFFu;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (bits & (1u << (2 * k))) u[k] &= 0xFFFF0000u;
        if (bits & (2u << (2 * k))) u[k] &= 0x0000FFFFu;
        const float x0 = __uint_as_float(u[k] << 16), x1 = __uint_as_float(u[k] & 0xFFFF0000u);
        ss0 = fmaf(x0, x0, ss0);
        ss1 = fmaf(x1, x1, ss1);
      }
      *reinterpret_cast<uint4*>(smem + L.a + hf * kTcARegion + r * 128 + ((c ^ (r & 7)) << 4)) =
          make_uint4(u[0], u[1], u[2], u[3]);
    }
    nrm_s[hf * kTcRows + r] = ss0 + ss1;
    // the outlier channels of this token, requested before the barrier
    float kout[kTcMaxOut];
#pragma unroll
    for (int o = 0; o < kTcMaxOut; ++o) kout[o] = (o < n_out && live) ? __bfloat162float(krow[idx_s[o]]) : 0.0f;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (tid == 0) {
      // P[128 x m] = A[128 x d] * S^T: d/16 MMAs per column block of at most 256
      for (int n0 = 0; n0 < m; n0 += 256) {
        const int n = min(256, m - n0);
        const uint32_t idesc = tc_idesc(n);
#pragma unroll
        for (int k = 0; k < kHeadDim / 16; ++k) {
          const uint32_t koff = (k & 3) * 32;  // 16 channels = 32 bytes inside a 128-byte row
          const uint64_t ad = tc_desc(a_base + (k >> 2) * kTcARegion + koff);
          const uint64_t bd = tc_desc(b_base + (k >> 2) * (m * 128) + n0 * 128 + koff);
          const uint32_t acc = k > 0 ? 1u : 0u;
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %4, 0;\n\t"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem + static_cast<uint32_t>(n0)),
              "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
              : "memory");
        }
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       tc_smem_u32(bar_mma))
                   : "memory");
    }
    // the next block's half row goes out now, behind this block's MMAs and epilogue
    if (item + 1 < item_end) key_half(item + 1, kh);

    // ---- norms: |k_in|^2 of both halves (fp32; an ambiguous fp16 rounding is
    // settled in fp64 from the A block), |k_out|^2 from the outlier channels
    const float nin32 = nrm_s[r] + nrm_s[kTcRows + r];
    float nout32 = 0.0f;
#pragma unroll
    for (int o = 0; o < kTcMaxOut; ++o) nout32 = fmaf(kout[o], kout[o], nout32);
    // |error| of an fp32 sum of n exact squares <= n 2^-24 of it (n = 128
    // bounds the summation tree of the two halves with room to spare)
    const float nin = sqrtf(nin32);
    int j = 0;
    unsigned char* tl = live ? tile_of(p.tiles, p.tl, bh, p.cap, pos, &j) : nullptr;
    if (live && hf == 0) {
      int h_in = tc_norm_fp16(nin32, 128.0f * 0x1p-24f);
      int h_out = tc_norm_fp16(nout32, 2.0f * kTcMaxOut * 0x1p-24f);
      if (h_in < 0) {
        double sd = 0.0;
        for (int c = 0; c < kHeadDim; ++c) {  // the masked row from the A block
          const int half = c >> 6, chunk = (c & 63) >> 3, within = c & 7;
          const unsigned short bits16 = *reinterpret_cast<const unsigned short*>(
              smem + L.a + half * kTcARegion + r * 128 + ((chunk ^ (r & 7)) << 4) + within * 2);
          const double x = __uint_as_float(static_cast<uint32_t>(bits16) << 16);
          sd = fma(x, x, sd);
        }
        h_in = __half_as_ushort(__double2half(sqrt(sd)));
      }
      if (h_out < 0) {
        double sd = 0.0;
#pragma unroll
        for (int o = 0; o < kTcMaxOut; ++o) sd = fma(static_cast<double>(kout[o]), static_cast<double>(kout[o]), sd);
        h_out = __half_as_ushort(__double2half(sqrt(sd)));
      }
      unsigned short* kn = reinterpret_cast<unsigned short*>(tl + p.tl.knorm) + 2 * j;
      kn[0] = static_cast<unsigned short>(h_in);
      kn[1] = static_cast<unsigned short>(h_out);
    }
    // ---- outlier sketch words hf, hf + 2, ...: n_out exact products per row,
    // summed in fp32 with |error| <= n_out 2^-24 sum |terms| <= n_out 2^-24
    // max_i |S_out[i, idx]| |k_out|; within twice that of zero, fp64 decides
    if (live) {
      const float thr_out = static_cast<float>(n_out) * 0x1p-23f * __uint_as_float(*so_max_bits) * sqrtf(nout32);
      for (int wo = hf; wo < wpo; wo += 2) {
        uint32_t word = n_out == 0 ? 0xFFFFFFFFu : 0u;  // no outlier channels: every projection is 0
#pragma unroll 4
        for (int bit = 0; bit < 32 && n_out > 0; ++bit) {
          const int i = 32 * wo + bit;
          const float4 s0 = reinterpret_cast<const float4*>(So + i * kTcMaxOut)[0];
          const float4 s1 = reinterpret_cast<const float4*>(So + i * kTcMaxOut)[1];
          const float sv[kTcMaxOut] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
          float y = 0.0f;
#pragma unroll
          for (int o = 0; o < kTcMaxOut; ++o) y = fmaf(sv[o], kout[o], y);  // kout is 0 past n_out
          bool sgn = y >= 0.0f;
          if (!(fabsf(y) > thr_out)) {
            double yd = 0.0;
#pragma unroll
            for (int o = 0; o < kTcMaxOut; ++o) yd = fma(static_cast<double>(sv[o]), static_cast<double>(kout[o]), yd);
            sgn = yd >= 0.0;
          }
          word |= (sgn ? 1u : 0u) << bit;
        }
        reinterpret_cast<uint32_t*>(tl + p.tl.kbits_out)[j * wpo + wo] = word;
      }
    }
    // ---- inlier sign words hf, hf + 2, ... from the accumulators
    bool mma_done = tc_wait(bar_mma, local & 1);
    if (!__syncthreads_and(mma_done)) {
      // give the MMAs a second bounded wait before their memory is released
      tc_wait(bar_mma, local & 1);
      ok = false;
    }
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const float thr = thr_rel * static_cast<float>(nin);
    // words wd and wd + 2 per round: two tensor-memory loads behind one wait
    for (int wd0 = hf; wd0 < wpt; wd0 += 4) {
      uint32_t va[32], vb[32];
      const int n_words = wd0 + 2 < wpt ? 2 : 1;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(32 * wd0);
      tc_ld32(va, taddr);
      if (n_words == 2) tc_ld32(vb, taddr + 64);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int half_w = 0; half_w < 2; ++half_w) {
        if (half_w >= n_words) break;
        const int wd = wd0 + 2 * half_w;
        const uint32_t* v = half_w == 0 ? va : vb;
        // bit = [y >= 0]: the complement of the sign bits, unless some |y| is
        // not clear of the guard band (then -0 and the near-zero entries are
        // decided one by one)
        float mn = fabsf(__uint_as_float(v[0]));
#pragma unroll
        for (int bit = 1; bit < 32; ++bit) mn = fminf(mn, fabsf(__uint_as_float(v[bit])));
        uint32_t neg = 0u;
#pragma unroll
        for (int bit = 0; bit < 32; ++bit) neg |= (v[bit] >> (31 - bit)) & (1u << bit);
        uint32_t word = ~neg, pending = 0u;
        if (!(mn > thr)) {
          word = 0u;
#pragma unroll
          for (int bit = 0; bit < 32; ++bit) {
            const float y = __uint_as_float(v[bit]);
            word |= (y >= 0.0f ? 1u : 0u) << bit;
            if (live && fabsf(y) < thr) pending |= 1u << bit;
          }
        }
        // near-zero projections: the exact sign from fp64, one entry at a time
        // for the whole warp (lane l sums channels 4l .. 4l+3)
        for (;;) {
          const uint32_t lanes = __ballot_sync(0xffffffffu, pending != 0u);
          if (lanes == 0u) break;
          const int src = __ffs(lanes) - 1;
          const int bsel = __shfl_sync(0xffffffffu, pending ? __ffs(pending) - 1 : 0, src);
          const int row = 32 * quarter + src, srow = 32 * wd + bsel;
          const int c0 = 4 * lane, half = c0 >> 6, chunk = (c0 & 63) >> 3, within = c0 & 7;
          const uint2 ka = *reinterpret_cast<const uint2*>(smem + L.a + half * kTcARegion + row * 128 +
                                                           ((chunk ^ (row & 7)) << 4) + within * 2);
          const uint2 sa = *reinterpret_cast<const uint2*>(smem + L.b + half * (m * 128) + srow * 128 +
                                                           ((chunk ^ (srow & 7)) << 4) + within * 2);
          double yd = static_cast<double>(__uint_as_float(ka.x << 16)) * __uint_as_float(sa.x << 16);
          yd = fma(static_cast<double>(__uint_as_float(ka.x & 0xFFFF0000u)), __uint_as_float(sa.x & 0xFFFF0000u), yd);
          yd = fma(static_cast<double>(__uint_as_float(ka.y << 16)), __uint_as_float(sa.y << 16), yd);
          yd = fma(static_cast<double>(__uint_as_float(ka.y & 0xFFFF0000u)), __uint_as_float(sa.y & 0xFFFF0000u), yd);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) yd += __shfl_xor_sync(0xffffffffu, yd, off);
          if (lane == src) {
            word = (word & ~(1u << bsel)) | ((yd >= 0.0 ? 1u : 0u) << bsel);
            pending &= ~(1u << bsel);
          }
        }
        if (live) reinterpret_cast<uint32_t*>(tl + p.tl.kbits)[j * wpt + wd] = word;
      }
    }
    if (!ok && live && hf == 0) {  // a timed-out wait: mark the token (NaN norms)
      unsigned short* kn = reinterpret_cast<unsigned short*>(tl + p.tl.knorm) + 2 * j;
      kn[0] = 0x7E00u;
      kn[1] = 0x7E00u;
    }
    // the next block rewrites the A block, the norms and the accumulators
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tcols) : "memory");
}

}  // namespace

// Whether the tensor-core sketch handles these keys (bf16, a full 128-token block or
// more, at most kTcMaxOut outlier channels).
bool sketch_keys_tc_applies(const KeysParams& p, qjl_dtype dt) {
  return dt == QJL_BF16 && p.T >= kTcRows && p.S_img != nullptr && p.m % 16 == 0 && p.m <= 512 &&
         p.n_out <= kTcMaxOut;
}

cudaError_t launch_sketch_keys_tc(const KeysParams& p, int num_sms, cudaStream_t s) {
  const TcSmem L(p.m, p.m_out, p.n_out);
  // CTAs per SM are capped through the shared-memory request so that their
  // tensor-memory columns fit the 512 of an SM (an allocation that cannot be
  // served would block).
  const int cols = tc_tmem_cols(p.m);
  const int max_ctas = 512 / cols;
  const int budget = 227 * 1024;
  size_t smem = static_cast<size_t>(L.total) + 1024;  // + alignment slack
  const size_t floor_bytes = static_cast<size_t>(budget / (max_ctas + 1) + 1024);
  if (smem < floor_bytes) smem = floor_bytes;
  if (smem > static_cast<size_t>(budget)) return cudaErrorInvalidConfiguration;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(sketch_keys_tc_kernel), smem);
  if (e != cudaSuccess) return e;
  const int tiles_per_bh = (p.T + kTcRows - 1) / kTcRows;
  const int64_t n_items64 = static_cast<int64_t>(p.B) * p.Hkv * tiles_per_bh;
  if (n_items64 > (1ll << 30)) return cudaErrorInvalidValue;
  const int n_items = static_cast<int>(n_items64);
  const int per_sm = static_cast<int>(budget / smem) < max_ctas ? static_cast<int>(budget / smem) : max_ctas;
  int grid = num_sms * (per_sm > 0 ? per_sm : 1);
  if (grid > n_items) grid = n_items;
  sketch_keys_tc_kernel<<<grid, kTcThreads, smem, s>>>(p, n_items, tiles_per_bh);
  return cudaGetLastError();
}

// The S image in the tcgen05 B-operand layout: two 64-channel halves, each
// m rows of 128 bytes; 16-byte chunk c of row n sits at chunk c ^ (n mod 8).
void tc_fill_s_image(const uint16_t* S, int m, uint16_t* img) {
  for (int n = 0; n < m; ++n)
    for (int c = 0; c < kHeadDim; ++c) {
      const int half = c / 64, chunk = (c % 64) / 8, within = c % 8;
      const size_t byte = static_cast<size_t>(half) * m * 128 + static_cast<size_t>(n) * 128 +
                          static_cast<size_t>((chunk ^ (n & 7)) * 16) + within * 2;
      img[byte / 2] = S[static_cast<size_t>(n) * kHeadDim + c];
    }
}

}  // namespace qjl
