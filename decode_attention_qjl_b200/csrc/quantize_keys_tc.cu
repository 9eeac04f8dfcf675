// QJL key sign sketch on the tensor cores (tcgen05), for bf16 keys in bulk.
//
// QJL summary (atlas.scime.ai), Approach: the key is multiplied by the random
// Gaussian JL matrix S and only sign(S k_in) is kept, plus the norm; the
// outlier channels get their own sketch sign(S_out k_out) and norm. For a
// block of 128 tokens of one (sequence, kv head) both projections are one
// dense product P = K [S_in; S_out]^T (128 x d times d x (m + m_out)), where
// S_in is S with the pair's outlier columns zeroed and S_out has its inlier
// columns zeroed, so that the unmasked key block serves both parts:
//   * the key block arrives by TMA (cp.async.bulk.tensor over a 4-d tensor map
//     of K with its own strides, 128-byte swizzle, tokens past T read as zero)
//     into one of three A buffers (two when [S; S_out] is large), so the next
//     blocks stream in while the current one is multiplied and read out;
//   * [S; S_out] is kept in shared memory in the 128-byte-swizzled K-major
//     layout of a tcgen05 B operand (qjl_init stores the image in global
//     memory; one bulk copy brings it in) and masked for the pair whenever
//     the pair changes;
//   * a producer warp issues the TMA loads and the MMAs: the columns of P in
//     passes of 128, each into one of four tensor-memory accumulators (bf16 x
//     bf16, fp32 accumulation), so the MMAs run up to four passes ahead of the
//     read-out;
//   * 16 epilogue warps, four per tensor-memory lane quarter: four threads per
//     token sum the exact squares of a quarter of its key's channels from the
//     A buffer (fp32; inlier channels through per-pair masks, the few outlier
//     ones one by one; the fp16 rounding of each norm is settled in fp64 when
//     the error bound does not fix it); then every warp reads one 32-column
//     word of each pass with tcgen05.ld (thread r gets token r's projections)
//     and packs the sign bits with one funnel shift per bit; the band test
//     takes the minimum |y| of the word first and goes bit by bit only when
//     it lies inside the band.
// A projection whose magnitude is at most d 2^-23 max_i |S_i| times the norm
// of its part (the error bound of an fp32 sum of the d exact bf16 x bf16
// products in any order, every addition truncated; by Cauchy-Schwarz) is
// recomputed in fp64 at the end of the block: exact products of the masked
// image row and the key row in the A buffer, eight lanes per entry, four
// entries at a time. So the bits equal the signs of the exact projections, as
// in the CUDA-core path.
// Work items (b, kv head, 128-token block) are contiguous ranges per
// persistent CTA (one per SM, 512 tensor-memory columns).
#include <cudaTypedefs.h>

#include "qjl_internal.cuh"

namespace qjl {
namespace {

constexpr int kTcRows = 128;                 // tokens per MMA block (M)
constexpr int kTcEpiWarps = 16;              // epilogue warps (4 per tensor-memory lane quadrant)
constexpr int kTcThreads = 32 * (kTcEpiWarps + 1);  // + the producer warp
constexpr int kTcHalf = kTcRows * 128;       // bytes of one 64-channel half of an A block
constexpr int kTcABytes = 2 * kTcHalf;       // one A block
constexpr int kTcPassCols = 128;             // accumulator columns per pass: one sign word per epilogue warp
constexpr int kTcBufs = 4;                   // tensor-memory accumulators (all 512 columns)
constexpr int kTcMaxPass = 5;                // passes per block at most (m + m_out <= 640; shared memory caps it lower)
constexpr uint64_t kTcWaitNs = 2000000000ull;

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
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(tc_smem_u32(bar)), "r"(parity), "r"(1000u)
      : "memory");
  return ok != 0;
}
__device__ __noinline__ bool tc_wait_slow(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = tc_timer();
  for (uint32_t n = 1;; ++n) {
    if (tc_try_wait(bar, parity)) return true;
    if ((n & 15u) == 0u && tc_timer() - t0 > kTcWaitNs) return false;
  }
}
// Wait for the phase with the given parity; false after kTcWaitNs.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) {
  return tc_try_wait(bar, parity) || tc_wait_slow(bar, parity);
}
__device__ __forceinline__ void tc_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc_smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(tc_smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(tc_smem_u32(bar))
               : "memory");
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
// Byte offset of channel c (bf16) of row `row` in a swizzled operand region of
// `rows` rows (two 64-channel halves of rows x 128 bytes).
__host__ __device__ inline int tc_swz(int rows, int row, int c) {
  return (c >> 6) * rows * 128 + row * 128 + ((((c & 63) >> 3) ^ (row & 7)) << 4) + (c & 7) * 2;
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

constexpr int kTcMaxA = 3;  // A buffers at most (fewer when [S; S_out] is large)

struct TcSmem {
  int na, a, b, nrm, pm, bars, misc, total;
  __host__ __device__ TcSmem(int rows, int n_a) {
    na = n_a;
    a = 0;                                  // A blocks [na] (1024-aligned)
    b = a + na * kTcABytes;                 // [S_in; S_out] image: rows x 256 bytes
    nrm = b + rows * kHeadDim * 2;          // float [na][4 channel quarters][128 rows][2]: sums of squares
    pm = nrm + na * 4 * kTcRows * 2 * 4;    // uint32 [epilogue warps][16]: inlier masks of channel pairs
    bars = pm + kTcEpiWarps * 16 * 4;       // a_full, a_free [kTcMaxA]; nrm_ready [kTcMaxA][4];
                                            // acc_full, acc_empty [kTcBufs]; img
    misc = bars + (6 * kTcMaxA + 2 * kTcBufs + 1) * 8;  // tensor-memory address, error flag
    total = misc + 16;
  }
};
// A buffers that fit beside the image of `rows` rows (0 if not even 2 fit).
__host__ __device__ inline int tc_num_a(int rows) {
  for (int na = kTcMaxA; na >= 2; --na)
    if (TcSmem(rows, na).total + 1024 <= 227 * 1024) return na;
  return 0;
}

// The outlier-channel mask (128 bits) of pair bh, the same in every lane.
__device__ __forceinline__ void tc_outlier_mask(const KeysParams& p, int64_t bh, uint32_t (&om)[4]) {
  const int lane = threadIdx.x & 31;
  const int c = lane < p.n_out ? min(max(p.idx[bh * p.n_out + lane], 0), kHeadDim - 1) : -1;
#pragma unroll
  for (int k = 0; k < 4; ++k) om[k] = __reduce_or_sync(0xffffffffu, c >= 0 && (c >> 5) == k ? 1u << (c & 31) : 0u);
}
// om[k] for a run-time k, by selects (an indexed read would put om in local memory).
__device__ __forceinline__ uint32_t tc_pick(const uint32_t (&om)[4], int k) {
  return k == 0 ? om[0] : k == 1 ? om[1] : k == 2 ? om[2] : om[3];
}

__global__ void __launch_bounds__(kTcThreads, 1)
    sketch_keys_tc_kernel(KeysParams p, const __grid_constant__ CUtensorMap tmap, int n_items, int tiles_per_bh,
                          int na) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // the swizzle of the MMA operands is a function of address bits 7..9: the
  // operand regions start on 1024-byte boundaries (1 KB is requested extra)
  unsigned char* smem = smem_raw + ((1024u - (tc_smem_u32(smem_raw) & 1023u)) & 1023u);
  const int m = p.m, m_out = p.m_out, rows = m + m_out;
  const int wpt = m >> 5, wpo = m_out >> 5, words = wpt + wpo;
  const int n_pass = (rows + kTcPassCols - 1) / kTcPassCols;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const TcSmem L(rows, na);
  float* nrm = reinterpret_cast<float*>(smem + L.nrm);
  uint64_t* a_full = reinterpret_cast<uint64_t*>(smem + L.bars);  // TMA of A buffer k landed
  uint64_t* a_free = a_full + kTcMaxA;     // the block in A buffer k is done with (MMAs and epilogue)
  uint64_t* nrm_ready = a_free + kTcMaxA;  // [k][q]: quarter q's norm sums of the block in A buffer k are in nrm[k]
  uint64_t* acc_full = nrm_ready + 4 * kTcMaxA;  // the pass in accumulator k is done
  uint64_t* acc_empty = acc_full + kTcBufs;      // accumulator k was read out
  uint64_t* img_bar = acc_empty + kTcBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  int* err = reinterpret_cast<int*>(tmem_slot + 1);

  if (tid == 0) {
    for (int k = 0; k < na; ++k) {
      tc_init(&a_full[k], 1);
      tc_init(&a_free[k], 1 + kTcEpiWarps);  // the MMA commit and every epilogue warp
      for (int q = 0; q < 4; ++q) tc_init(&nrm_ready[4 * k + q], kTcEpiWarps / 4);  // the quarter's four warps
    }
    for (int k = 0; k < kTcBufs; ++k) {
      tc_init(&acc_full[k], 1);
      tc_init(&acc_empty[k], kTcEpiWarps);
    }
    tc_init(img_bar, 1);
    *err = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tc_smem_u32(tmem_slot)),
                 "r"(kTcBufs * kTcPassCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  const uint32_t a_base = tc_smem_u32(smem + L.a), b_base = tc_smem_u32(smem + L.b);
  // this CTA's blocks are a contiguous range, so that consecutive blocks
  // mostly share their (b, kv head) and its outlier channels
  const int per = n_items / gridDim.x, extra = n_items % gridDim.x;
  const int item_begin = blockIdx.x * per + min(static_cast<int>(blockIdx.x), extra);
  const int n_local = per + (static_cast<int>(blockIdx.x) < extra ? 1 : 0);

  if (warp == kTcEpiWarps) {
    // ============================================================ producer
    bool ok = true;
    int64_t cur_bh = -1;
    int passes = 0;  // MMA passes issued
    int n_img = 0;   // image loads (phases of img_bar)
    auto tma_a = [&](int i) {  // the key block of local item i into A buffer i % na
      const int item = item_begin + i;
      const int64_t bh = item / tiles_per_bh;
      const int b = static_cast<int>(bh / p.Hkv), h = static_cast<int>(bh % p.Hkv);
      const int y = (item % tiles_per_bh) * kTcRows;
      uint64_t* bar = &a_full[i % na];
      const uint32_t dst = a_base + (i % na) * kTcABytes;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_smem_u32(bar)), "r"(kTcABytes)
                   : "memory");
#pragma unroll
      for (int half = 0; half < 2; ++half)
        asm volatile(
            "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
            "%5}], [%6];" ::"r"(dst + half * kTcHalf),
            "l"(&tmap), "r"(64 * half), "r"(y), "r"(h), "r"(b), "r"(tc_smem_u32(bar))
            : "memory");
    };
    if (lane == 0)
      for (int i = 0; i < na - 1 && i < n_local; ++i) tma_a(i);
    for (int i = 0; i < n_local && ok; ++i) {
      const int item = item_begin + i;
      const int64_t bh = item / tiles_per_bh;
      if (bh != cur_bh) {  // the image masked for this pair's outlier channels
        // the previous block is released by the MMAs and every epilogue warp
        // (whose exact fallback reads the image)
        if (lane == 0 && i >= 1)
          if (!tc_wait(&a_free[(i - 1) % na], ((i - 1) / na) & 1)) ok = false;
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        if (!ok) break;
        if (lane == 0) {
          const uint32_t bytes = static_cast<uint32_t>(rows) * kHeadDim * 2;
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tc_smem_u32(img_bar)),
                       "r"(bytes)
                       : "memory");
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(b_base),
              "l"(p.S_img), "r"(bytes), "r"(tc_smem_u32(img_bar))
              : "memory");
        }
        uint32_t om[4];
        tc_outlier_mask(p, bh, om);
        const int c_l = lane < p.n_out ? min(max(p.idx[bh * p.n_out + lane], 0), kHeadDim - 1) : 0;
        // lane l edits 16-byte chunk l % 16 of the S_out rows: its 8 outlier bits
        const uint32_t keep = (tc_pick(om, (lane & 15) >> 2) >> (8 * (lane & 3))) & 0xFFu;
        bool got = true;
        if (lane == 0) got = tc_wait(img_bar, n_img & 1);
        ++n_img;
        ok = __shfl_sync(0xffffffffu, got, 0) != 0;
        cur_bh = bh;
        if (!ok) break;
        // S_in rows lose the outlier channels, S_out rows keep only them
        unsigned char* img = smem + L.b;
        for (int o = 0; o < p.n_out; ++o) {
          const int c = __shfl_sync(0xffffffffu, c_l, o);
          for (int row = lane; row < m; row += 32) *reinterpret_cast<uint16_t*>(img + tc_swz(rows, row, c)) = 0;
        }
        if (keep != 0xFFu)
          for (int e = lane; e < m_out * (kHeadDim / 8); e += 32) {
            uint4* q = reinterpret_cast<uint4*>(img + tc_swz(rows, m + (e >> 4), 8 * (e & 15)));
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (keep != 0u) {
              w = *q;
              const uint32_t k0 = (keep & 1u ? 0xFFFFu : 0u) | (keep & 2u ? 0xFFFF0000u : 0u);
              const uint32_t k1 = (keep & 4u ? 0xFFFFu : 0u) | (keep & 8u ? 0xFFFF0000u : 0u);
              const uint32_t k2 = (keep & 16u ? 0xFFFFu : 0u) | (keep & 32u ? 0xFFFF0000u : 0u);
              const uint32_t k3 = (keep & 64u ? 0xFFFFu : 0u) | (keep & 128u ? 0xFFFF0000u : 0u);
              w.x &= k0; w.y &= k1; w.z &= k2; w.w &= k3;
            }
            *q = w;
          }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor-core reads
        __syncwarp();
      }
      if (lane == 0) {
        if (!tc_wait(&a_full[i % na], (i / na) & 1)) ok = false;
        for (int pass = 0; pass < n_pass && ok; ++pass, ++passes) {
          const int buf = passes % kTcBufs;
          if (passes >= kTcBufs && !tc_wait(&acc_empty[buf], (passes / kTcBufs - 1) & 1)) {
            ok = false;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const int n0 = pass * kTcPassCols, n = min(kTcPassCols, rows - n0);
          const uint32_t idesc = tc_idesc(n);
          const uint32_t a_buf = a_base + (i % na) * kTcABytes;
#pragma unroll
          for (int k = 0; k < kHeadDim / 16; ++k) {
            const uint32_t koff = (k & 3) * 32;  // 16 channels = 32 bytes inside a 128-byte row
            const uint64_t ad = tc_desc(a_buf + (k >> 2) * kTcHalf + koff);
            const uint64_t bd = tc_desc(b_base + (k >> 2) * (rows * 128) + n0 * 128 + koff);
            const uint32_t acc = k > 0 ? 1u : 0u;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem + buf * kTcPassCols),
                "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                : "memory");
          }
          tc_commit(&acc_full[buf]);
        }
        if (ok) tc_commit(&a_free[i % na]);  // the block's MMAs no longer read its A buffer
      }
      ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
      // block i + na - 1 streams in behind this one (its buffer held block i - 1)
      if (i + na - 1 < n_local) {
        if (lane == 0) {
          if (i >= 1 && !tc_wait(&a_free[(i - 1) % na], ((i - 1) / na) & 1)) ok = false;
          if (ok) tma_a(i + na - 1);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
      }
    }
    // drain: the last MMAs and copies complete before the CTA may release its memory
    if (lane == 0) {
      for (int q = passes > kTcBufs ? passes - kTcBufs : 0; q < passes; ++q)
        tc_wait(&acc_full[q % kTcBufs], (q / kTcBufs) & 1);
      for (int i = n_local > na ? n_local - na : 0; i < n_local; ++i) tc_wait(&a_full[i % na], (i / na) & 1);
      if (!ok) atomicExch(err, 1);
    }
  } else {
    // ============================================================ epilogue
    const int quarter = warp & 3, sub = warp >> 2;  // tensor-memory lanes 32 quarter .., channel quarter sub
    const int r = 32 * quarter + lane;               // token row of this thread
    // d 2^-23 max_i |S_i|: the bound of an fp32 sum of d exact products in any
    // order with truncating additions (half the context's band), and 2^-10 more
    // for the fp32 rounding of the norm and of the band itself
    const float thr_rel = 0.5005f * p.guard_tc;
    // this warp's inlier masks of its 16 channel pairs (bf16 pairs of channels 32 sub ..)
    uint32_t* pmask = reinterpret_cast<uint32_t*>(smem + L.pm) + 16 * warp;
    bool ok = true;
    int64_t cur_bh = -1;
    uint32_t om[4] = {0u, 0u, 0u, 0u};
    uint32_t mw = 0u, ol4 = 0u;  // outlier bits of channels 32 sub .. +31, and of 4 lane .. 4 lane + 3
    int passes = 0;
    int tile = item_begin % tiles_per_bh, pos0 = 0;  // block of the pair; first position of sequence b
    int ab = 0;          // A buffer of block i: i % na
    uint32_t aph = 0u;   // its phase parity: (i / na) & 1
    for (int i = 0; i < n_local; ++i, ++tile, ab = ab + 1 == na ? 0 : ab + 1, aph ^= ab == 0 ? 1u : 0u) {
      if (tile == tiles_per_bh) tile = 0;
      const int64_t bh = cur_bh < 0 ? item_begin / tiles_per_bh : cur_bh + (tile == 0 ? 1 : 0);
      if (bh != cur_bh) pos0 = p.t_start ? p.t_start[bh / p.Hkv] : 0;
      const int t = tile * kTcRows + r;
      const int pos = pos0 + t;
      const bool live = t < p.T && pos >= 0 && pos < p.cap;
      int j = 0;
      unsigned char* tl = live ? tile_of(p.tiles, p.tl, bh, p.cap, pos, &j) : nullptr;
      if (bh != cur_bh) {
        tc_outlier_mask(p, bh, om);
        mw = tc_pick(om, sub);
        ol4 = (tc_pick(om, lane >> 3) >> ((4 * lane) & 31)) & 0xFu;
        if (lane < 16)
          pmask[lane] = ((mw >> (2 * lane)) & 1u ? 0u : 0x0000FFFFu) | ((mw >> (2 * lane + 1)) & 1u ? 0u : 0xFFFF0000u);
        __syncwarp();
        cur_bh = bh;
      }
      const unsigned char* A = smem + L.a + ab * kTcABytes;
      // ---- norms of token r: this thread sums the exact squares of channels
      // 32 sub .. 32 sub + 31 in fp32: the inlier ones through the pair masks,
      // the (few) outlier ones one by one
      {
        if (ok && !tc_wait(&a_full[ab], aph)) ok = false;
        float s_in = 0.0f, s_out = 0.0f;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 8 channels (16 bytes) per chunk
          const uint4 w = *reinterpret_cast<const uint4*>(A + tc_swz(kTcRows, r, 32 * sub + 8 * ch));
          const uint4 mk = reinterpret_cast<const uint4*>(pmask)[ch];
          const uint32_t u[4] = {w.x & mk.x, w.y & mk.y, w.z & mk.z, w.w & mk.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float lo = __uint_as_float(u[k] << 16), hi = __uint_as_float(u[k] & 0xFFFF0000u);
            s_in = fmaf(lo, lo, s_in);
            s_in = fmaf(hi, hi, s_in);
          }
        }
        for (uint32_t rest = mw; rest != 0u; rest &= rest - 1u) {
          const int c = 32 * sub + __ffs(rest) - 1;
          const float x = __uint_as_float(
              static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(A + tc_swz(kTcRows, r, c))) << 16);
          s_out = fmaf(x, x, s_out);
        }
        float* np = nrm + (ab * 4 + sub) * kTcRows * 2 + 2 * r;
        np[0] = s_in;
        np[1] = s_out;
        __syncwarp();
        if (lane == 0) tc_arrive(&nrm_ready[4 * ab + quarter]);  // this warp's part of the sums is in place
      }
      if (ok && !tc_wait(&nrm_ready[4 * ab + quarter], aph)) ok = false;
      float n2_in = 0.0f, n2_out = 0.0f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 pq = *reinterpret_cast<const float2*>(nrm + (ab * 4 + q) * kTcRows * 2 + 2 * r);
        n2_in += pq.x;
        n2_out += pq.y;
      }
      const float thr_in = thr_rel * sqrtf(n2_in), thr_out = thr_rel * sqrtf(n2_out);
      if (sub == 0) {  // warp-uniform: these four warps write the norms
        // |error| of an fp32 sum of n exact squares <= n 2^-24 of it (n = 128
        // bounds the four partial sums and their total with room to spare)
        int h_in = tc_norm_fp16(n2_in, 128.0f * 0x1p-24f), h_out = tc_norm_fp16(n2_out, 128.0f * 0x1p-24f);
        // rows whose fp16 norm the bound leaves open: fp64 from the key row in
        // the A buffer, one row at a time for the whole warp (lane l squares
        // channels 4l .. 4l+3)
        uint32_t open = __ballot_sync(0xffffffffu, live && (h_in < 0 || h_out < 0));
        while (open != 0u) {
          const int src = __ffs(open) - 1;
          open &= open - 1u;
          const uint2 ka = *reinterpret_cast<const uint2*>(A + tc_swz(kTcRows, 32 * quarter + src, 4 * lane));
          const double x0 = __uint_as_float(ka.x << 16), x1 = __uint_as_float(ka.x & 0xFFFF0000u);
          const double x2 = __uint_as_float(ka.y << 16), x3 = __uint_as_float(ka.y & 0xFFFF0000u);
          double d_in = 0.0, d_out = 0.0;
          (ol4 & 1u ? d_out : d_in) += x0 * x0;
          (ol4 & 2u ? d_out : d_in) += x1 * x1;
          (ol4 & 4u ? d_out : d_in) += x2 * x2;
          (ol4 & 8u ? d_out : d_in) += x3 * x3;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            d_in += __shfl_xor_sync(0xffffffffu, d_in, off);
            d_out += __shfl_xor_sync(0xffffffffu, d_out, off);
          }
          if (lane == src) {
            if (h_in < 0) h_in = __half_as_ushort(__double2half(sqrt(d_in)));
            if (h_out < 0) h_out = __half_as_ushort(__double2half(sqrt(d_out)));
          }
        }
        if (live) {
          unsigned short* kn = reinterpret_cast<unsigned short*>(tl + p.tl.knorm) + 2 * j;
          kn[0] = static_cast<unsigned short>(ok ? h_in : 0x7E00u);
          kn[1] = static_cast<unsigned short>(ok ? h_out : 0x7E00u);
        }
      }
      // ---- sign words: this warp takes word wl of every pass (a short last
      // pass leaves some warps idle, rotating from block to block); bit =
      // [y >= 0] is the complement of the sign bit, and every |y| <= thr (-0
      // among them, and all of a zero key) stays pending for the exact sign
      const int wl = (sub + i) & 3;
      uint32_t word[kTcMaxPass], pend[kTcMaxPass];
#pragma unroll
      for (int s = 0; s < kTcMaxPass; ++s) {
        word[s] = 0u;
        pend[s] = 0u;
      }
#pragma unroll
      for (int s = 0; s < kTcMaxPass; ++s) {
        if (s >= n_pass) break;
        const int buf = passes % kTcBufs;
        if (ok && !tc_wait(&acc_full[buf], (passes / kTcBufs) & 1)) ok = false;
        ok = __all_sync(0xffffffffu, ok);  // the warp takes the branch below as one
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int wd = 4 * s + wl;  // word of [S_in; S_out] rows (inlier words first)
        if (wd < words && ok) {
          uint32_t v[32];
          tc_ld32(v, tmem + (static_cast<uint32_t>(32 * quarter) << 16) + static_cast<uint32_t>(buf * kTcPassCols + 32 * wl));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          const float thr = wd < wpt ? thr_in : thr_out;
          // a shift register, one funnel shift per bit: the sign bit of y; then
          // the word's smallest |y| (and, inside the band, the sign bit of
          // thr - |y| per bit: set when |y| > thr)
          uint32_t neg = 0u;
#pragma unroll
          for (int bit = 31; bit >= 0; --bit) neg = __funnelshift_l(v[bit], neg, 1);
          float mn[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) mn[k] = fminf(fabsf(__uint_as_float(v[2 * k])), fabsf(__uint_as_float(v[2 * k + 1])));
#pragma unroll
          for (int w2 = 8; w2 > 0; w2 >>= 1)
#pragma unroll
            for (int k = 0; k < w2; ++k) mn[k] = fminf(mn[k], mn[k + w2]);
          word[s] = ~neg;
          uint32_t pd = 0u;
          // the exact per-bit band test only for a word whose smallest |y| is
          // inside the band; a NaN projection needs a non-finite key, whose
          // norm, and so thr, is NaN or infinite, and takes this path too
          if (live && !(mn[0] > thr)) {
            uint32_t far = 0u;
#pragma unroll
            for (int bit = 31; bit >= 0; --bit)
              far = __funnelshift_l(__float_as_uint(thr - fabsf(__uint_as_float(v[bit]))), far, 1);
            pd = ~far;
          }
          pend[s] = pd;
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) tc_arrive(&acc_empty[buf]);
        ++passes;
      }
      // ---- pending entries: the exact sign from fp64, four entries at a time:
      // lanes 8g .. 8g+7 take the first pending entry of the g-th lane that has
      // one, each summing 16 channels of the masked image row and of the key
      // row in the A buffer
      for (;;) {
        uint32_t any = 0u;
#pragma unroll
        for (int s = 0; s < kTcMaxPass; ++s) any |= pend[s];
        const uint32_t lanes = __ballot_sync(0xffffffffu, any != 0u);
        if (lanes == 0u) break;
        const int grp = lane >> 3;
        int src = 0, mine = -1;  // this group's entry lane; the group that takes this lane's entry
        uint32_t rest = lanes;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int l = rest != 0u ? __ffs(rest) - 1 : -1;
          if (g == grp && l >= 0) src = l;
          if (l == lane) mine = g;
          rest &= rest - 1u;
        }
        int entry = 0;  // 32 slot + bit of this lane's first pending entry
#pragma unroll
        for (int s = kTcMaxPass - 1; s >= 0; --s)
          if (pend[s] != 0u) entry = 32 * s + __ffs(pend[s]) - 1;
        const int e = __shfl_sync(0xffffffffu, entry, src);
        const int srow = 32 * (4 * (e >> 5) + wl) + (e & 31), row = 32 * quarter + src;
        const int c0 = 16 * (lane & 7);
        double y0 = 0.0, y1 = 0.0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint4 sa = *reinterpret_cast<const uint4*>(smem + L.b + tc_swz(rows, srow, c0 + 8 * half));
          const uint4 ka = *reinterpret_cast<const uint4*>(A + tc_swz(kTcRows, row, c0 + 8 * half));
          const uint32_t su[4] = {sa.x, sa.y, sa.z, sa.w}, ku[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // bf16 x bf16 products are exact in fp32: one conversion each
            y0 += static_cast<double>(__fmul_rn(__uint_as_float(ku[k] << 16), __uint_as_float(su[k] << 16)));
            y1 += static_cast<double>(__fmul_rn(__uint_as_float(ku[k] & 0xFFFF0000u), __uint_as_float(su[k] & 0xFFFF0000u)));
          }
        }
        double yd = y0 + y1;
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) yd += __shfl_xor_sync(0xffffffffu, yd, off);
        yd = __shfl_sync(0xffffffffu, yd, 8 * (mine < 0 ? 0 : mine));
        if (mine >= 0) {
          const uint32_t set = yd >= 0.0 ? ~0u : 0u;
#pragma unroll
          for (int s = 0; s < kTcMaxPass; ++s) {  // masks, not an indexed update (which would go to local memory)
            const uint32_t bit = (entry >> 5) == s ? 1u << (entry & 31) : 0u;
            word[s] = (word[s] & ~bit) | (set & bit);
            pend[s] &= ~bit;
          }
        }
      }
      if (live) {
#pragma unroll
        for (int s = 0; s < kTcMaxPass; ++s) {
          const int wd = 4 * s + wl;
          if (s < n_pass && wd < words) {
            if (wd < wpt)
              reinterpret_cast<uint32_t*>(tl + p.tl.kbits)[j * wpt + wd] = word[s];
            else
              reinterpret_cast<uint32_t*>(tl + p.tl.kbits_out)[j * wpo + (wd - wpt)] = word[s];
          }
        }
      }
      // this warp is done with the block: its A buffer, norm sums and (for the
      // producer's image reload) the image rows may be reused
      __syncwarp();
      if (lane == 0) tc_arrive(&a_free[ab]);
      if (!ok && live && sub == 0) {  // a timed-out wait: mark the token (NaN norms)
        unsigned short* kn = reinterpret_cast<unsigned short*>(tl + p.tl.knorm) + 2 * j;
        kn[0] = 0x7E00u;
        kn[1] = 0x7E00u;
      }
    }
    if (!ok && lane == 0) atomicExch(err, 1);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcBufs * kTcPassCols) : "memory");
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

// Whether the tensor-core sketch handles these keys: bf16, a full 128-token
// block or more, strides the tensor map can describe, and [S; S_out] plus two
// A blocks in shared memory.
bool sketch_keys_tc_applies(const KeysParams& p, qjl_dtype dt) {
  if (dt != QJL_BF16 || p.T < kTcRows || p.S_img == nullptr) return false;
  if ((p.B > 1 && p.sb == 0) || (p.Hkv > 1 && p.sh == 0)) return false;  // broadcast batches or heads
  if (p.m + p.m_out > kTcMaxPass * kTcPassCols) return false;
  return tc_num_a(p.m + p.m_out) >= 2 && tc_encode_fn() != nullptr;
}

cudaError_t launch_sketch_keys_tc(const KeysParams& p, int num_sms, cudaStream_t s) {
  const int na = tc_num_a(p.m + p.m_out);
  if (na < 2) return cudaErrorInvalidConfiguration;
  const TcSmem L(p.m + p.m_out, na);
  // the kernel takes 512 tensor-memory columns: one CTA per SM, which a
  // shared-memory request of more than half the SM's also enforces
  size_t smem = static_cast<size_t>(L.total) + 1024;  // + alignment slack
  if (smem < 116 * 1024) smem = 116 * 1024;
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(sketch_keys_tc_kernel), smem);
  if (e != cudaSuccess) return e;
  // 4-d tensor map of K: (channel, token, kv head, sequence), element strides
  // as given (16-byte multiples, checked by the caller); a dimension of extent
  // 1 gets a harmless stride
  CUtensorMap tmap;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(p.T),
                              static_cast<cuuint64_t>(p.Hkv), static_cast<cuuint64_t>(p.B)};
  const cuuint64_t row = static_cast<cuuint64_t>(p.st) * 2;
  const cuuint64_t sh = p.Hkv > 1 ? static_cast<cuuint64_t>(p.sh) * 2 : row * p.T;
  const cuuint64_t sb = p.B > 1 ? static_cast<cuuint64_t>(p.sb) * 2 : sh * p.Hkv;
  const cuuint64_t strides[3] = {row, sh, sb};
  const cuuint32_t box[4] = {64, kTcRows, 1, 1};
  const cuuint32_t estride[4] = {1, 1, 1, 1};
  PFN_cuTensorMapEncodeTiled_v12000 enc = tc_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const CUresult cr = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.K), dims, strides, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const int tiles_per_bh = (p.T + kTcRows - 1) / kTcRows;
  const int64_t n_items64 = static_cast<int64_t>(p.B) * p.Hkv * tiles_per_bh;
  if (n_items64 > (1ll << 30)) return cudaErrorInvalidValue;
  const int n_items = static_cast<int>(n_items64);
  const int grid = num_sms < n_items ? num_sms : n_items;
  sketch_keys_tc_kernel<<<grid, kTcThreads, smem, s>>>(p, tmap, n_items, tiles_per_bh, na);
  return cudaGetLastError();
}

// The image in the tcgen05 B-operand layout: two 64-channel halves, each
// `rows` rows of 128 bytes; 16-byte chunk c of row n sits at chunk c ^ (n mod 8).
void tc_fill_s_image(const uint16_t* S, int rows, uint16_t* img) {
  for (int n = 0; n < rows; ++n)
    for (int c = 0; c < kHeadDim; ++c) img[tc_swz(rows, n, c) / 2] = S[static_cast<size_t>(n) * kHeadDim + c];
}

}  // namespace qjl
