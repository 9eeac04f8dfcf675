// QJL decode attention.
//
// QJL summary (atlas.scime.ai), Approach: the query is JL-projected WITHOUT
// quantisation and a cached token's score is the unbiased asymmetric estimator
//   s_t = sqrt(pi/2)/m * |k_in| * <S q_in, sign(S k_in)>
//       + sqrt(pi/2)/m_out * |k_out| * <S_out q_out, sign(S_out k_out)>.
// With packed bits, <sq, sign> = 2 * sum_{bit set} sq_i - sum_i sq_i.
// p = online softmax of sm_scale * s; o = sum_t p_t (code_t * scale_t + zero_t).
//
// One launch per call: decode_kernel, persistent (at most one CTA per SM).
// The CTAs never wait for one another.
//
// Query blocks. Before a work item's tiles can be scored, the CTA builds the
//    item's query block in shared memory: the G = Hq/Hkv queries of its
//    (b, kv head) projected on the tensor cores (sq = S q_in, S_out q_out,
//    bf16 operands, fp32 accumulation) and turned into integers:
//    x_i = rint(sq_i * 2^F) with |x_i| < 2^29 (a power-of-two scale per head
//    and part), then x'_i = round(x_i / 2^(i mod 8)) so that the sign bit of
//    row i, which sits at bit (i mod 8) of its byte, can enter the MMA as the
//    byte value 2^(i mod 8) without being shifted down. x' is stored as four
//    int8 limbs per entry, already in the per-lane B fragment order of the
//    score MMA, followed by F and sum_i 2^(i mod 8) x'_i. The consumer and
//    combiner warps build the first item's block together; the combiner warp
//    builds each later item's block while the consumers work on the item
//    before it (two buffers).
//
// Main loop. Each CTA walks the work items (b, kv head, token split)
//    blockIdx.x, blockIdx.x + gridDim.x, ...
//    * The producer warp streams each item's
//      cache tiles (64 tokens each: sign words, outlier sign words, norms,
//      value codes, scale/zero) into a shared-memory ring, several consecutive
//      tiles per cp.async.bulk copy (mbarrier completion, L2 evict-first
//      policy, no multicast).
//    * The consumer warps (14, 10 or 6 by G, so that the register file holds
//      all warps) take the item's tiles round-robin. Per tile:
//      - scores on the tensor cores: the A fragment of an int8 m16n8k32 MMA is
//        the sign word masked to one bit per byte (byte values 2^(i mod 8)); one
//        N-tile of 8 columns carries the 4 limbs of 2 heads; the limb sums are
//        exact in int32 and combined in fp32;
//      - online softmax per head over the tile with one lane per token (exp2
//        with log2(e) folded into the scale);
//      - values on the tensor cores, 16 tokens at a time: A = value codes of 16
//        dims of one group (ldmatrix.trans of the staged tile, nibbles turned
//        into fp16 integers by a lop3), B = p * scale split into fp16 hi and lo
//        columns (22 significant bits), fp32 accumulation; the zero-point term
//        sum_t p_t * zero_t is accumulated per group on CUDA cores.
//    * After an item each consumer warp writes its partial (max, sum, o) to
//      shared memory; the combiner warp merges them and writes the item's
//      partial (or the output), and the last item of a (b, kv head), found
//      with an atomic ticket, merges the splits, all off the consumers' path.
//      There is no CTA-wide barrier in the loop.
// Every wait (mbarrier, ring sequence) is bounded in time; on a
// timeout the kernel writes NaN to the outputs it owns and returns.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

constexpr int kTT = kDecodeTileTokens;  // tokens per tile (the cache capacity is a multiple)
constexpr int kMaxStages = 8;           // ring stages of kStageTiles tiles (the count is set per launch)
constexpr int kNQ = kDecodeQBuffers;    // query-block buffers (by item parity)
constexpr int kPartStride = kHeadDim + 4 + 2;  // per (warp, head) partial: o[d], zero sums[4], max, sum
constexpr int kSStride = 72;            // floats per head in a warp's score / probability buffer (padded)
constexpr int kWStride = 36;            // words per (head, limb) in a warp's value B-operand buffer (padded)
constexpr int kSmemBudget = 227 * 1024;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait

// Launch shape by heads per kv head.
template <int G>
struct Shape {
  static constexpr int NC = G <= 2 ? 14 : (G == 4 ? 10 : 6);  // consumer warps
  static constexpr int THREADS = 32 * (NC + 2);  // + producer warp + combiner warp
  static constexpr int NTS = (G + 1) / 2;  // score N-tiles: 2 heads x 4 limbs
  static constexpr int NTV = (G + 3) / 4;  // value N-tiles: 4 heads x (hi, lo)
  static constexpr int NB = G <= 2 ? 2 : 1;  // combine buffers
  static constexpr int FRAG_BUDGET = G <= 2 ? 24 : (G == 4 ? 48 : 96);  // query fragment registers
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer() - t0 > kWaitLimitNs) return false;
  }
  return true;
}
// Wait until a ring slot's published fill number reaches `fill`; false after kWaitLimitNs.
__device__ __noinline__ bool seq_wait(const int* seq, int fill) {
  const volatile int* v = seq;
  if (*v >= fill) {
    __threadfence_block();
    return true;
  }
  const uint64_t t0 = global_timer();
  while (*v < fill) {
    __nanosleep(64);  // leave the issue slots to the other warps of the SM
    if (global_timer() - t0 > kWaitLimitNs) return false;
  }
  __threadfence_block();
  return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// The same with an L2 cache policy (createpolicy), for the cache stream.
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// L2 policy for data read once: evicted first, so that the small data every
// call reuses (sketch matrices, queries, workspace, code) stays in L2.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// int8 MMA: D(16x8, s32) += A(16x32, u8) * B(32x8, s8)
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// fp16 MMA: D(16x8, f32) += A(16x16, f16) * B(16x8, f16)
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(row_addr));
}
// fp16 integers from nibbles without shifting them down: a nibble in bits 0-3
// of each half becomes 1024 + n, one in bits 4-7 becomes 64 + n (the fp16
// exponent is chosen so that the mantissa step equals 1); the subtraction
// leaves n exactly.
__device__ __forceinline__ uint32_t nib_lo_h2(uint32_t x) {
  uint32_t r, out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x000F000Fu), "r"(0x64006400u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(out) : "r"(r), "r"(0x64006400u));
  return out;
}
__device__ __forceinline__ uint32_t nib_hi_h2(uint32_t x) {
  uint32_t r, out;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x00F000F0u), "r"(0x54005400u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(out) : "r"(r), "r"(0x54005400u));
  return out;
}

// int8 limb l (0 = low) of x = L3 * 2^24 + L2 * 2^16 + L1 * 2^8 + L0, every limb in [-128, 127].
__device__ __forceinline__ int limb_of(int x, int l) {
  const int l0 = static_cast<int8_t>(x & 0xFF);
  const int x1 = (x - l0) >> 8;
  const int l1 = static_cast<int8_t>(x1 & 0xFF);
  const int x2 = (x1 - l1) >> 8;
  const int l2 = static_cast<int8_t>(x2 & 0xFF);
  const int l3 = (x2 - l2) >> 8;
  return l == 0 ? l0 : (l == 1 ? l1 : (l == 2 ? l2 : l3));
}

// Shared-memory scratch of the query-block builds (bytes): per build parity
// and (head, part) the sum of 2^(i mod 8) x'_i (int64) and max |sq| (float
// bits), both zero at rest: the finishing lanes of build j reset the slots of
// parity j % 2 after its last barrier, before they enter build j + 1 (whose
// barriers every other warp must pass before it can reach build j + 2).
__host__ __device__ inline int build_scratch_bytes(int G, int m, int m_out) {
  return 2 * (G * 2 * 8 + G * 2 * 4);
}

// ------------------------------------------------------------------ layouts
// A ring stage holds kStageTiles consecutive cache tiles exactly as they lie in
// global memory (TileLayout offsets inside each tile).
struct Smem {
  // byte offsets from the dynamic shared-memory base
  int stages, bars, qbuf, comb, sbuf, wbuf, bscr, misc, total, qblock;
  __host__ __device__ Smem(int G, int NC, int NB, int m, int m_out, int nstage) {
    const TileLayout tl = tile_layout(m, m_out);
    qblock = static_cast<int>(decode_qblock_bytes(G, m, m_out));
    stages = 0;
    // full, empty [kMaxStages]; qfull, qfree [kNQ]; cfree, cfull [2]; image (+1 slot of padding)
    bars = stages + nstage * kStageTiles * tl.bytes;
    qbuf = bars + (2 * kMaxStages + 2 * kNQ + 6) * 8;  // query blocks [kNQ] (bulk-copy targets)
    comb = qbuf + kNQ * qblock;                        // fp32 [NB][NC][G][kPartStride]
    sbuf = comb + NB * NC * G * kPartStride * 4;       // fp32 [NC][G][kSStride]
    wbuf = sbuf + NC * G * kSStride * 4;               // u32 [NC][2G][kWStride]
    bscr = wbuf + NC * 2 * G * kWStride * 4;           // query-block build scratch
    misc = bscr + ((build_scratch_bytes(G, m, m_out) + 15) & ~15);  // fill sequence [kMaxStages], flags
    total = misc + (kMaxStages + 3) * 4;
  }
  // every section starts on a 16-byte boundary (bulk copies, vector accesses)
  __host__ __device__ bool aligned() const {
    return ((stages | bars | qbuf | comb | sbuf | wbuf | bscr | misc | qblock) & 15) == 0;
  }
};
// Ring stages that fit the shared-memory budget (at most kMaxStages, 0 if not even 2 fit).
template <int G>
int decode_nstage(int m, int m_out) {
  for (int n = kMaxStages; n >= 2; --n)
    if (Smem(G, Shape<G>::NC, Shape<G>::NB, m, m_out, n).total <= kSmemBudget) return n;
  return 0;
}


// ------------------------------------------------------------------ query blocks
// Query block of one (b, kv head) (bytes), built in shared memory by the CTA
// that needs it:
//   fragment word (t * KK + kk) * 2 + h of lane l at word index (...) * 32 + l:
//   for lane (r, q) (column r of N-tile t: head 2t + r/4, limb r % 4), byte j
//   holds that limb of x'[head] at sketch row 32kk + 2q + h + 8j (kk < m/32:
//   inlier rows, then outlier rows); then int32 F[G][2] and int64 sum[G][2]
//   (inlier, outlier part).
__device__ __forceinline__ void named_sync(int threads) {
  asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}

// The fixed-point exponent of one (head, part) from the float bits of max|sq|:
// F = 29 - e for max|sq| in [2^(e-1), 2^e), so that |sq_i| 2^F < 2^29; 0 when
// the part is all zero. A maximum below the normal range is treated as 2^-126.
__device__ __forceinline__ int qblock_exponent(unsigned int mx_bits) {
  if (mx_bits == 0u) return 0;
  const int E = max(static_cast<int>((mx_bits >> 23) & 0xFF), 1);  // max|sq| < 2^(E - 126)
  return 155 - E;  // in [-99, 154]
}
// 2^F as two normal floats whose product it is (2^F alone overflows for F > 127);
// sq * s.x * s.y is then exact.
__device__ __forceinline__ float2 qblock_scale(int F) {
  const int f1 = min(F, 127), f2 = F - f1;  // f2 in [0, 27]
  return make_float2(__int_as_float((f1 + 127) << 23), __int_as_float((f2 + 127) << 23));
}

// One query-block build: the query block of pair bh into dst (shared or
// global memory), run by the nw warps wi = 0 .. nw-1 (one named barrier
// inside); the caller then runs build_finish after a barrier over the same
// warps.
// Sketch row i (inlier rows 0 .. m-1, then outlier rows) is the dot product of
// row i of S (or of S_out) with the query restricted to the inlier (or to the
// outlier) channels, on the tensor cores: sq[rows x G] = S[rows x d] q[d x G]
// as bf16 m16n8k16 MMAs with fp32 accumulation. The A fragments come from
// S_frag (S and S_out in the per-lane fragment order): from its shared-memory
// copy `simg` when there is one, else from global memory. The B fragments are
// the query (an fp32 query split into bf16 hi and lo parts, each its own MMA).
// Warp wi takes the 32-row words kk = wi, wi + nw, ...: the two 16-row tiles
// of a word, kept in registers while the warps exchange their maxima (F per
// (head, part) from max|sq|), then x = rint(sq 2^F) (an exact scaling) and
// x' = round(x / 2^(i mod 8)) in the accumulator lanes, moved into the
// fragment lanes by shuffles and packed as int8 limbs; the word's sums of
// 2^(i mod 8) x'_i are added to sums[head][part] (shared atomics).
// The global loads of a build, issued ahead of it: this lane's query values
// (head r, channels 16 ks + 2q + {0, 1, 8, 9}) and one outlier index per lane.
struct QLoad {
  float qv[kHeadDim / 16][4];
  int c_idx;
};
template <int G>
__device__ __forceinline__ void load_query(const DecodeParams& p, int64_t bh, QLoad& ql) {
  constexpr int KS = kHeadDim / 16;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2, q = lane & 3;
  const int b = static_cast<int>(bh / p.Hkv), hk = static_cast<int>(bh % p.Hkv);
  const int64_t qrow = (static_cast<int64_t>(b) * p.Hq + hk * G + (r < G ? r : 0)) * kHeadDim;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int c0 = 16 * ks + 2 * q;
    if (p.q_fp32) {
      const float2 v0 = *reinterpret_cast<const float2*>(static_cast<const float*>(p.Q) + qrow + c0);
      const float2 v1 = *reinterpret_cast<const float2*>(static_cast<const float*>(p.Q) + qrow + c0 + 8);
      ql.qv[ks][0] = v0.x; ql.qv[ks][1] = v0.y; ql.qv[ks][2] = v1.x; ql.qv[ks][3] = v1.y;
    } else {
      const __nv_bfloat162 v0 =
          *reinterpret_cast<const __nv_bfloat162*>(static_cast<const __nv_bfloat16*>(p.Q) + qrow + c0);
      const __nv_bfloat162 v1 =
          *reinterpret_cast<const __nv_bfloat162*>(static_cast<const __nv_bfloat16*>(p.Q) + qrow + c0 + 8);
      ql.qv[ks][0] = __low2float(v0); ql.qv[ks][1] = __high2float(v0);
      ql.qv[ks][2] = __low2float(v1); ql.qv[ks][3] = __high2float(v1);
    }
    if (r >= G) ql.qv[ks][0] = ql.qv[ks][1] = ql.qv[ks][2] = ql.qv[ks][3] = 0.0f;
  }
  ql.c_idx = lane < p.n_out ? min(max(p.idx[bh * p.n_out + lane], 0), kHeadDim - 1) : -1;
}

template <int G, int WMAX>
__device__ __forceinline__ void build_qblock(const DecodeParams& p, const QLoad& ql, unsigned char* dst,
                                             unsigned long long* sums, unsigned int* maxes, const uint4* simg, int wi,
                                             int nw) {
  constexpr int NTS = (G + 1) / 2;
  constexpr int KS = kHeadDim / 16;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2, q = lane & 3;
  const int m = p.m, m_out = p.m_out, n_out = p.n_out;
  const int wpt = m >> 5, wpo = m_out >> 5, KK = wpt + wpo;

  const float (&qv)[KS][4] = ql.qv;
  const int c_idx = ql.c_idx;
  uint32_t om[4];  // outlier channels of this pair as a 128-bit mask
#pragma unroll
  for (int k = 0; k < 4; ++k)
    om[k] = __reduce_or_sync(0xffffffffu, c_idx >= 0 && (c_idx >> 5) == k ? 1u << (c_idx & 31) : 0u);
  // channel 16 ks + 2q + (e & 1) + 8 (e >> 1) is an outlier (its mask word is om[ks / 2])
  auto qo = [&](int ks, int e) {
    const int c = 16 * ks + 2 * q + (e & 1) + 8 * (e >> 1);
    return ((om[ks >> 1] >> (c & 31)) & 1u) != 0u;
  };
  // pass 1: the words of this warp (at most WMAX) on the tensor cores, kept in
  // registers; this warp's max |sq| per (head 2q + e, part)
  float acc[WMAX][2][4];
  float mx[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};  // [e][part]
#pragma unroll
  for (int w = 0; w < WMAX; ++w) {
    const int kk = wi + w * nw;
    if (kk >= KK) break;
    const int part = kk < wpt ? 0 : 1;
    const int mt = part ? (m + 32 * (kk - wpt)) / 16 : 2 * kk;  // the word's first 16-row tile
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[w][u][k] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      // B[k][n] = query of head n at channel 16 ks + k, this part's channels only
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = qo(ks, e) == (part == 1) ? qv[ks][e] : 0.0f;
      // An fp32 query is the exact sum of three bf16 limbs (8 + 8 + 8
      // significant bits: each remainder is exact in fp32 and has at most 8
      // bits left after two roundings), each its own MMA with exact products.
      uint32_t lb[3][2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float x0 = v[2 * half], x1 = v[2 * half + 1];
#pragma unroll
        for (int l = 0; l < 3; ++l) {
          const __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
          lb[l][half] = *reinterpret_cast<const uint32_t*>(&hb);
          x0 -= __low2float(hb);
          x1 -= __high2float(hb);
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int64_t ai = (static_cast<int64_t>(mt + u) * KS + ks) * 32 + lane;
        const uint4 a = simg ? simg[ai] : __ldg(p.S_frag + ai);
        mma_bf16(acc[w][u], a, lb[0][0], lb[0][1]);
        if (p.q_fp32) {
          mma_bf16(acc[w][u], a, lb[1][0], lb[1][1]);
          mma_bf16(acc[w][u], a, lb[2][0], lb[2][1]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = fmaxf(fmaxf(fabsf(acc[w][0][e]), fabsf(acc[w][0][2 + e])), fmaxf(fabsf(acc[w][1][e]), fabsf(acc[w][1][2 + e])));
      if (part)
        mx[e][1] = fmaxf(mx[e][1], v);
      else
        mx[e][0] = fmaxf(mx[e][0], v);
    }
  }
  // the maxima of all warps: [warp][head][part]
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      float v = mx[e][part];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
      if (r == 0 && 2 * q + e < G && v > 0.0f) atomicMax(&maxes[(2 * q + e) * 2 + part], __float_as_uint(v));
    }
  named_sync(32 * nw);
  // F of the heads 2q, 2q + 1 that this lane holds as an accumulator lane, per part
  int Fa[2][2];
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      Fa[e][part] = 2 * q + e < G ? qblock_exponent(maxes[(2 * q + e) * 2 + part]) : 0;
    }
  if (wi == 0 && lane < 2 * G) {  // F per (head, part)
    reinterpret_cast<int*>(dst + 4 * NTS * KK * 64)[lane] = qblock_exponent(maxes[lane]);
  }

  // pass 2: fixed point, sums and fragment words of this warp's words
#pragma unroll
  for (int w = 0; w < WMAX; ++w) {
    const int kk = wi + w * nw;
    if (kk >= KK) break;
    const int part = kk < wpt ? 0 : 1;
    // accumulator lane (r, q): rows r, r + 8 of tiles u = 0, 1 (word rows 16u + r (+8)),
    // heads 2q + e in acc[u][e] (row r) and acc[u][2 + e] (row r + 8); i mod 8 = r
    int xp[2][4];
    long long sx[2] = {0, 0};  // per head 2q + e
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 sc = qblock_scale(part ? Fa[e][1] : Fa[e][0]);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int x = __float2int_rn(acc[w][u][2 * k + e] * sc.x * sc.y);
          const int v = r ? (x + (1 << (r - 1))) >> r : x;  // round half up
          xp[u][2 * k + e] = v;
          sx[e] += static_cast<long long>(v) << r;
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      sx[e] += __shfl_xor_sync(0xffffffffu, sx[e], 4);
      sx[e] += __shfl_xor_sync(0xffffffffu, sx[e], 8);
      sx[e] += __shfl_xor_sync(0xffffffffu, sx[e], 16);
      if (r == 0 && 2 * q + e < G) atomicAdd(&sums[(2 * q + e) * 2 + part], static_cast<unsigned long long>(sx[e]));
    }
    // fragment word (t, kk, h) of lane (r, q): head 2t + r/4, limb r % 4, byte j = row 2q + h + 8j
    // of the word, held by accumulator lane 4 (2q + h) + head/2 (tile j/2, register 2 (j%2) + head%2)
    uint32_t* fr = reinterpret_cast<uint32_t*>(dst);
#pragma unroll
    for (int t = 0; t < NTS; ++t) {
      const int head = 2 * t + (r >> 2), limb = r & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int src = 4 * (2 * q + h) + (min(head, G - 1) >> 1);
        uint32_t v = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int u = j >> 1, k = j & 1;
          const int x0 = __shfl_sync(0xffffffffu, xp[u][2 * k], src);
          const int x1 = __shfl_sync(0xffffffffu, xp[u][2 * k + 1], src);
          const int x = (head & 1) ? x1 : x0;
          v |= (static_cast<uint32_t>(limb_of(x, limb)) & 0xFFu) << (8 * j);
        }
        fr[((t * KK + kk) * 2 + h) * 32 + lane] = head < G ? v : 0u;
      }
    }
  }
}

// After build_qblock and a barrier over its warps: the (head, part) sums of
// the block, by lanes 0 .. 2G-1 of one warp, which also reset the scratch.
template <int G>
__device__ __forceinline__ void build_finish(const DecodeParams& p, unsigned char* dst, unsigned long long* sums,
                                             unsigned int* maxes) {
  constexpr int NTS = (G + 1) / 2;
  const int lane = threadIdx.x & 31;
  const int KK = (p.m >> 5) + (p.m_out >> 5);
  if (lane < 2 * G) {
    reinterpret_cast<long long*>(dst + 4 * NTS * KK * 64 + 8 * G)[lane] = static_cast<long long>(sums[lane]);
    sums[lane] = 0ull;
    maxes[lane] = 0u;
  }
}

// ------------------------------------------------------------------ work items
// Item i = split + splits * (kv head + Hkv * b): a token range of one (b, kv head).
struct Item {
  int b, hk, split, t0, t1;
  int n_tile;   // 64-token tiles
  int n_stage;  // ring stages (kStageTiles tiles each, the last one possibly shorter)
  int64_t bh;
};
__device__ __forceinline__ Item item_of(const DecodeParams& p, int i) {
  Item it;
  it.split = i % p.splits;
  const int rest = i / p.splits;
  it.hk = rest % p.Hkv;
  it.b = rest / p.Hkv;
  it.bh = static_cast<int64_t>(it.b) * p.Hkv + it.hk;
  int len = p.seqlens ? p.seqlens[it.b] : p.T;
  len = max(0, min(len, p.T));
  it.t0 = it.split * p.chunk;
  it.t1 = min(len, it.t0 + p.chunk);
  it.n_tile = it.t1 > it.t0 ? (it.t1 - it.t0 + kTT - 1) / kTT : 0;
  it.n_stage = (it.n_tile + kStageTiles - 1) / kStageTiles;
  return it;
}

// ------------------------------------------------------------------ main kernel
// WPT_MAX / WPO_MAX bound the inlier / outlier sign words per token; with
// EXACT they are the exact counts, so that every word loop is fully static.
template <int G, int WPT_MAX, int WPO_MAX, bool FR, bool EXACT>
__global__ void __launch_bounds__(Shape<G>::THREADS, 1) decode_kernel(DecodeParams p) {
  constexpr int NC = Shape<G>::NC, NTS = Shape<G>::NTS, NTV = Shape<G>::NTV, NB = Shape<G>::NB;
  constexpr int WPO_A = WPO_MAX > 0 ? WPO_MAX : 1;
  constexpr int FRI = FR ? WPT_MAX : 1, FRO = FR ? WPO_A : 1;  // query fragments held in registers
  constexpr int SU = 1;  // score sub-tiles per pass (2 measured no faster and costs registers)
  extern __shared__ __align__(128) unsigned char smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = EXACT ? 32 * WPT_MAX : p.m, m_out = EXACT ? 32 * WPO_MAX : p.m_out;
  const int wpt = m >> 5, wpo = m_out >> 5, KK = wpt + wpo;
  const int n_items = p.B * p.Hkv * p.splits;
  const int nstage = p.nstage;
  const Smem L(G, NC, NB, m, m_out, nstage);
  const TileLayout ST = p.tl;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kMaxStages;
  uint64_t* qfull = empty + kMaxStages;
  uint64_t* qfree = qfull + kNQ;
  uint64_t* cfree = qfree + kNQ;
  uint64_t* cfull = cfree + 2;
  int* fill_seq = reinterpret_cast<int*>(smem + L.misc);  // [kMaxStages]: fill last issued into each ring slot
  int* flag = fill_seq + kMaxStages;                      // error flag
  int* p0_done = flag + 1;                                // every query block of this CTA is built
  int* q0_back = flag + 2;                                // the first build's query loads are back
  uint64_t* img_bar = cfull + 2;
  unsigned char* bscr = smem + L.bscr;
  // S_frag is staged once in the tail of the ring, which the producer fills
  // last, when it fits there
  const int ring_bytes = nstage * kStageTiles * ST.bytes;
  const int img_bytes = (m + m_out) * 2 * kHeadDim;
  const bool use_img = img_bytes <= ring_bytes;
  const int img_off = use_img ? ring_bytes - img_bytes : ring_bytes;  // 16-byte aligned
  const int n_local = n_items > static_cast<int>(blockIdx.x)
                          ? (n_items - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                          : 0;  // items of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstage; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kStageTiles);  // one arrival per tile (the producer stands in for missing tiles)
      fill_seq[s] = -1;
    }
    for (int k = 0; k < kNQ; ++k) {
      mbar_init(&qfull[k], 1);   // the builder (first kNQ items) or the producer's copy
      mbar_init(&qfree[k], NC);  // every consumer warp releases every query block
    }
    for (int k = 0; k < NB; ++k) {
      mbar_init(&cfree[k], 1);   // the combiner releases the combine buffer
      mbar_init(&cfull[k], NC);  // every consumer warp posts its partial
    }
    mbar_init(img_bar, 1);
    *flag = 0;
    *p0_done = 0;
    *q0_back = 0;
    for (int e = 0; e < build_scratch_bytes(G, m, m_out) / 4; ++e) reinterpret_cast<unsigned int*>(bscr)[e] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (use_img) {
      mbar_arrive_expect_tx(img_bar, static_cast<uint32_t>(img_bytes));
      bulk_g2s(smem + L.stages + img_off, p.S_frag, static_cast<uint32_t>(img_bytes), img_bar);
    }
  }
  __syncthreads();

  if (warp != NC && n_local > 0) {
    // ============================================================ query blocks
    // The consumer and combiner warps build the query blocks of all items of
    // this CTA together (one warp alone would take far longer: the build is
    // a chain of short latency-bound steps): the first kNQ into shared
    // memory, the rest into the workspace (the producer brings them in
    // later). The blocks depend on no other CTA. The producer streams cache
    // stages meanwhile, into the ring slots that the S image leaves free.
    const int wi = warp < NC ? warp : NC;
    const uint4* simg = use_img ? reinterpret_cast<const uint4*>(smem + L.stages + img_off) : nullptr;
    unsigned long long* sums0 = reinterpret_cast<unsigned long long*>(bscr);  // [parity][G][2]
    unsigned int* maxes0 = reinterpret_cast<unsigned int*>(sums0 + 4 * G);     // [parity][G][2]
    constexpr int WMAX = (WPT_MAX + WPO_A + NC) / (NC + 1);  // words per building warp, at most
    // each build's query loads go out one build ahead (the first during the image copy)
    QLoad cur;
    load_query<G>(p, item_of(p, blockIdx.x).bh, cur);
    if (warp == 0) {  // behind the ring fill these loads would wait several microseconds
      float z = cur.c_idx;
#pragma unroll
      for (int ks = 0; ks < kHeadDim / 16; ++ks) z += cur.qv[ks][0] + cur.qv[ks][1] + cur.qv[ks][2] + cur.qv[ks][3];
      asm volatile("" ::"f"(z));  // the flag goes up only once every loaded value is in
      __syncwarp();
      if (lane == 0) *reinterpret_cast<volatile int*>(q0_back) = 1;
    }
    if (use_img && !mbar_wait(img_bar, 0)) atomicExch(flag, 1);
    for (int j = 0; j < n_local; ++j) {
      QLoad nxt;
      if (j + 1 < n_local) load_query<G>(p, item_of(p, blockIdx.x + (j + 1) * gridDim.x).bh, nxt);
      const int i = blockIdx.x + j * gridDim.x;
      unsigned char* dst = j < kNQ ? smem + L.qbuf + j * L.qblock
                                   : p.qblock + static_cast<int64_t>(i - kNQ * static_cast<int>(gridDim.x)) * p.qblock_bytes;
      unsigned long long* sums = sums0 + (j & 1) * 2 * G;
      unsigned int* maxes = maxes0 + (j & 1) * 2 * G;
      build_qblock<G, WMAX>(p, cur, dst, sums, maxes, simg, wi, NC + 1);
      named_sync(32 * (NC + 1));
      if (warp == NC + 1) {  // the builder's last step
        build_finish<G>(p, dst, sums, maxes);
        __syncwarp();
        if (j < kNQ && lane == 0) mbar_arrive(&qfull[j]);
      }
      if (j + 1 < n_local) cur = nxt;
    }
    if (n_local > kNQ) asm volatile("fence.proxy.async.global;" ::: "memory");  // blocks read by bulk copies
    named_sync(32 * (NC + 1));
    if (warp == NC + 1 && lane == 0) {
      __threadfence_block();
      *reinterpret_cast<volatile int*>(p0_done) = 1;  // the image is free, the stored blocks are ready
    }
  }

  if (warp == NC) {
    // ============================================================ producer
    // (one lane: a blocking mbarrier wait stalls its whole warp, so no other
    // role shares this warp)
    if (lane == 0) {
      // the first query block's loads go out ahead of the ring fill
      bool ok = seq_wait(q0_back, 1), built = false;
      const int img_slot = img_off / (kStageTiles * ST.bytes);  // first ring slot that overlaps the image
      const uint64_t stream_policy = evict_first_policy();
      int gs = 0;  // stages issued so far (ring slot gs % nstage, fill gs / nstage)
      int il = 0;  // local item counter
      const int64_t tiles_per_slab = p.cap / kTT;
      for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x, ++il) {
        const Item it = item_of(p, i);
        if (il >= kNQ) {  // this item's query block comes from the workspace, ahead of its tiles
          const int kb = il % kNQ;
          if (!built && !seq_wait(p0_done, 1)) {
            ok = false;
            break;
          }
          built = true;
          if (!mbar_wait(&qfree[kb], ((il / kNQ) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&qfull[kb], L.qblock);
          bulk_g2s(smem + L.qbuf + kb * L.qblock,
                   p.qblock + static_cast<int64_t>(i - kNQ * static_cast<int>(gridDim.x)) * p.qblock_bytes, L.qblock,
                   &qfull[kb]);
        }
        // the item's tiles are consecutive in global memory
        const unsigned char* g_tile =
            p.tiles + (it.bh * tiles_per_slab + it.t0 / kTT) * static_cast<int64_t>(ST.bytes);
        for (int s = 0; s < it.n_stage && ok; ++s) {
          const int slot = gs % nstage;
          if (gs >= nstage && !mbar_wait(&empty[slot], ((gs / nstage) - 1) & 1)) {
            ok = false;
            break;
          }
          if (gs < nstage && slot >= img_slot && !built) {  // the image is read until the blocks are built
            if (!seq_wait(p0_done, 1)) {
              ok = false;
              break;
            }
            built = true;
          }
          // Consumers skip stages that other warps consume, so a parity wait alone
          // could match an older phase: they first wait for this fill number.
          __threadfence_block();
          *reinterpret_cast<volatile int*>(&fill_seq[slot]) = gs / nstage;
          const int nt = min(kStageTiles, it.n_tile - s * kStageTiles);
          const uint32_t bytes = static_cast<uint32_t>(nt * ST.bytes);
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_g2s_hint(smem + L.stages + slot * kStageTiles * ST.bytes,
                        g_tile + static_cast<int64_t>(s) * kStageTiles * ST.bytes, bytes, &full[slot], stream_policy);
          // a short stage: arrive for the tiles no consumer will release
          if (nt < kStageTiles) mbar_arrive_cnt(&empty[slot], kStageTiles - nt);
          ++gs;
        }
      }
      // Drain: every copy issued here lands before the CTA may exit.
      for (int g = gs > nstage ? gs - nstage : 0; g < gs; ++g)
        if (!mbar_wait(&full[g % nstage], (g / nstage) & 1)) ok = false;
      for (int k = il > 2 * kNQ ? il - kNQ : kNQ; k < il; ++k)
        if (!mbar_wait(&qfull[k % kNQ], (k / kNQ) & 1)) ok = false;
      if (!ok) atomicExch(flag, 1);
    }
    return;
  }
  if (warp == NC + 1) {
    // ============================================================ combiner
    // Merges the consumer warps' partials of each item, off the consumers'
    // critical path, and merges the splits of a (b, kv head).
    {
      bool failed = false;
      int il = 0;
      for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++il) {
        const Item it = item_of(p, i);
        const int cb = il % NB;
        if (!failed && !mbar_wait(&cfull[cb], (il / NB) & 1)) {
          failed = true;
          atomicExch(flag, 1);
        }
        __threadfence_block();
        failed |= *reinterpret_cast<volatile int*>(flag) != 0;
        const float* cbuf = reinterpret_cast<const float*>(smem + L.comb) + cb * NC * G * kPartStride;
        const int hq0 = it.hk * G;
        for (int e = lane; e < G * kHeadDim; e += 32) {
          const int j = e / kHeadDim, c = e % kHeadDim;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < NC; ++w) M = fmaxf(M, cbuf[(w * G + j) * kPartStride + kHeadDim + 4]);
          float Lsum = 0.0f, ov = 0.0f;
          if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NC; ++w) {
              const float* pw = cbuf + (w * G + j) * kPartStride;
              const float mw = pw[kHeadDim + 4];
              if (mw == -INFINITY) continue;
              const float f = exp2f(mw - M);
              Lsum += pw[kHeadDim + 5] * f;
              ov += (pw[c] + pw[kHeadDim + (c >> 5)]) * f;
            }
          }
          if (failed) ov = __int_as_float(0x7fc00000);  // NaN marks a timed-out wait
          const int64_t orow = static_cast<int64_t>(it.b) * p.Hq + hq0 + j;
          if (p.splits == 1) {
            p.O[orow * kHeadDim + c] = failed ? ov : (Lsum > 0.0f ? ov / Lsum : 0.0f);
          } else {
            const int64_t prow = orow * p.splits + it.split;
            p.part_o[prow * kHeadDim + c] = ov;
            if (c == 0) {
              p.part_ml[2 * prow] = M;
              p.part_ml[2 * prow + 1] = Lsum;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&cfree[cb]);
        if (p.splits > 1) {
          // ---- the last item of this (b, kv head) merges the splits
          __threadfence();
          __syncwarp();
          int merge = 0;
          if (lane == 0) merge = atomicAdd(p.tickets + it.bh, 1) == p.splits - 1;
          merge = __shfl_sync(0xffffffffu, merge, 0);
          if (merge) {
            __threadfence();
            // per head: the splits' maximum over the lanes, then 4 channels per
            // lane with the splits' loads independent of one another
            for (int j = 0; j < G; ++j) {
              const int64_t orow = static_cast<int64_t>(it.b) * p.Hq + hq0 + j;
              float M = -INFINITY;
              for (int sp = lane; sp < p.splits; sp += 32) M = fmaxf(M, __ldcg(p.part_ml + 2 * (orow * p.splits + sp)));
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
              float Lsum = 0.0f;
              float4 ov = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              bool nan = false;
#pragma unroll 4
              for (int sp = 0; sp < p.splits; ++sp) {
                const int64_t prow = orow * p.splits + sp;
                const float4 os = __ldcg(reinterpret_cast<const float4*>(p.part_o + prow * kHeadDim) + lane);
                const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml) + prow);
                nan |= os.x != os.x || os.y != os.y || os.z != os.z || os.w != os.w;
                const float f = M == -INFINITY || ml.x == -INFINITY ? 0.0f : exp2f(ml.x - M);
                Lsum = fmaf(ml.y, f, Lsum);
                ov.x = fmaf(os.x, f, ov.x);
                ov.y = fmaf(os.y, f, ov.y);
                ov.z = fmaf(os.z, f, ov.z);
                ov.w = fmaf(os.w, f, ov.w);
              }
              const bool pos = Lsum > 0.0f;
              const float4 o = nan ? make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                                 __int_as_float(0x7fc00000), __int_as_float(0x7fc00000))
                                   : make_float4(pos ? ov.x / Lsum : 0.0f, pos ? ov.y / Lsum : 0.0f,
                                                 pos ? ov.z / Lsum : 0.0f, pos ? ov.w / Lsum : 0.0f);
              reinterpret_cast<float4*>(p.O + orow * kHeadDim)[lane] = o;
            }
            if (lane == 0) p.tickets[it.bh] = 0;  // leave the counter at zero for the next call
          }
        }
      }
    }
    return;
  }

  // ============================================================== consumers
  const int r = lane >> 2, q = lane & 3;     // MMA fragment coordinates
  const int tp = lane & 7, gq = lane >> 3;   // value B-operand builder: token pair, value group
  const uint32_t mask_a0 = 0x01010101u << (2 * q), mask_a2 = mask_a0 << 1;
  // score MMA columns 2q, 2q+1 hold limbs 0,1 (q even) or 2,3 (q odd) of head 2t + q/2
  const float limb_w = (q & 1) ? 65536.0f : 1.0f;
  float* Sw = reinterpret_cast<float*>(smem + L.sbuf) + warp * G * kSStride;        // [G][kSStride]
  uint32_t* Ww = reinterpret_cast<uint32_t*>(smem + L.wbuf) + warp * 2 * G * kWStride;  // [2G][kWStride]
  const float c_in0 = kSqrtHalfPi / static_cast<float>(m);
  const float c_out0 = m_out > 0 ? kSqrtHalfPi / static_cast<float>(m_out) : 0.0f;

  uint32_t fri[NTS][FRI][2], fro[NTS][FRO][2];
  float cin[NTS], cout[NTS], xin[NTS], xout[NTS];
  int gs_base = 0;  // ring stages of the items before the current one
  int gt_base = 0;  // tiles of the items before the current one (tiles go round-robin to the warps)
  int il = 0;
  bool ok = true;

  for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++il) {
    const Item it = item_of(p, i);
    const int qb = il % kNQ, cb = il % NB;
    // ---- query block of this item
    if (ok && !mbar_wait(&qfull[qb], (il / kNQ) & 1)) ok = false;
    const int first = (warp - gt_base % NC + NC) % NC;  // this warp's first tile of the item
    const bool works = ok && first < it.n_tile;
    const uint32_t* qfr = reinterpret_cast<const uint32_t*>(smem + L.qbuf + qb * L.qblock) + lane;
    if (works) {
      if (FR) {
#pragma unroll
        for (int t = 0; t < NTS; ++t) {
#pragma unroll
          for (int kk = 0; kk < FRI; ++kk)
#pragma unroll
            for (int h = 0; h < 2; ++h) fri[t][kk][h] = kk < wpt ? qfr[((t * KK + kk) * 2 + h) * 32] : 0u;
#pragma unroll
          for (int kk = 0; kk < FRO; ++kk)
#pragma unroll
            for (int h = 0; h < 2; ++h) fro[t][kk][h] = kk < wpo ? qfr[((t * KK + wpt + kk) * 2 + h) * 32] : 0u;
        }
      }
      const unsigned char* tail = smem + L.qbuf + qb * L.qblock + 4 * NTS * KK * 64;
      const int* Fs = reinterpret_cast<const int*>(tail);
      const long long* sums = reinterpret_cast<const long long*>(tail + 8 * G);
#pragma unroll
      for (int t = 0; t < NTS; ++t) {
        const int hd = min(2 * t + (q >> 1), G - 1);
        cin[t] = ldexpf(c_in0, -Fs[2 * hd]);
        cout[t] = ldexpf(c_out0, -Fs[2 * hd + 1]);
        xin[t] = __ll2float_rn(sums[2 * hd]);
        xout[t] = __ll2float_rn(sums[2 * hd + 1]);
      }
    }
    if (FR) {  // fragments are in registers: release the query block now
      __syncwarp();
      if (lane == 0) mbar_arrive(&qfree[qb]);
    }

    // ---- running state of this warp for this item
    float run_m[G], run_l[G], zacc[G];  // run_m warp-uniform; run_l and zacc per lane
#pragma unroll
    for (int h = 0; h < G; ++h) {
      run_m[h] = -INFINITY;
      run_l[h] = 0.0f;
      zacc[h] = 0.0f;
    }
    // value accumulators: [group][dim pair][N-tile][fragment]: thread (r, q) holds
    // dims 32g + 4r + 2P (regs 0, 1: hi, lo) and 32g + 4r + 2P + 1 (regs 2, 3) of head 4v + q
    float vacc[4][2][NTV][4];
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int P = 0; P < 2; ++P)
#pragma unroll
        for (int v = 0; v < NTV; ++v)
#pragma unroll
          for (int k = 0; k < 4; ++k) vacc[g][P][v][k] = 0.0f;

    for (int s = first; works && ok && s < it.n_tile; s += NC) {
      const int gs = gs_base + s / kStageTiles;
      const int slot = gs % nstage;
      if (!seq_wait(&fill_seq[slot], gs / nstage) || !mbar_wait(&full[slot], (gs / nstage) & 1)) {
        ok = false;
        break;
      }
      const unsigned char* stg = smem + L.stages + (slot * kStageTiles + s % kStageTiles) * ST.bytes;
      const int tile0 = it.t0 + s * kTT;            // first token of the tile
      const int n_valid = min(kTT, it.t1 - tile0);  // >= 1
      // ---------------- scores of the 64 tokens (4 sub-tiles of 16 rows) into Sw,
      // SU sub-tiles per pass so that their MMA chains interleave (the pass
      // loop stays rolled: the unrolled tile body would not fit the
      // instruction cache)
#pragma unroll 1
      for (int u0 = 0; u0 < 4; u0 += SU) {
        int ai[SU][NTS][4], ao[SU][NTS][4];
#pragma unroll
        for (int j = 0; j < SU; ++j)
#pragma unroll
          for (int t = 0; t < NTS; ++t)
#pragma unroll
            for (int k = 0; k < 4; ++k) ai[j][t][k] = ao[j][t][k] = 0;
        // row r of sub-tile u0 + j at wr + 16 j wpt, row r + 8 a further 8 wpt
        const uint32_t* wr = reinterpret_cast<const uint32_t*>(stg + ST.kbits) + (16 * u0 + r) * wpt;
        auto score_word = [&](int j, int kk, uint32_t wa, uint32_t wb) {
          const uint32_t a0 = wa & mask_a0, a2 = wa & mask_a2, a1 = wb & mask_a0, a3 = wb & mask_a2;
#pragma unroll
          for (int t = 0; t < NTS; ++t) {
            const uint32_t b0 = FR ? fri[t][FR ? kk : 0][0] : qfr[((t * KK + kk) * 2 + 0) * 32];
            const uint32_t b1 = FR ? fri[t][FR ? kk : 0][1] : qfr[((t * KK + kk) * 2 + 1) * 32];
            mma_u8s8(ai[j][t], a0, a1, a2, a3, b0, b1);
          }
        };
        if ((wpt & 3) == 0) {  // rows are whole 16-byte vectors
#pragma unroll
          for (int k4 = 0; k4 < WPT_MAX; k4 += 4) {
            if (k4 < wpt) {
              uint4 va[SU], vb[SU];
#pragma unroll
              for (int j = 0; j < SU; ++j) {
                va[j] = *reinterpret_cast<const uint4*>(wr + 16 * j * wpt + k4);
                vb[j] = *reinterpret_cast<const uint4*>(wr + (16 * j + 8) * wpt + k4);
              }
#pragma unroll
              for (int j = 0; j < SU; ++j) score_word(j, k4 + 0, va[j].x, vb[j].x);
#pragma unroll
              for (int j = 0; j < SU; ++j) score_word(j, k4 + 1, va[j].y, vb[j].y);
#pragma unroll
              for (int j = 0; j < SU; ++j) score_word(j, k4 + 2, va[j].z, vb[j].z);
#pragma unroll
              for (int j = 0; j < SU; ++j) score_word(j, k4 + 3, va[j].w, vb[j].w);
            }
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < WPT_MAX; ++kk)
            if (kk < wpt)
#pragma unroll
              for (int j = 0; j < SU; ++j) score_word(j, kk, wr[16 * j * wpt + kk], wr[(16 * j + 8) * wpt + kk]);
        }
        if (WPO_MAX > 0) {
          const uint32_t* wo = reinterpret_cast<const uint32_t*>(stg + ST.kbits_out) + (16 * u0 + r) * wpo;
#pragma unroll
          for (int ko = 0; ko < WPO_A; ++ko) {
            if (ko < wpo) {
#pragma unroll
              for (int j = 0; j < SU; ++j) {
                const uint32_t wa = wo[16 * j * wpo + ko], wb = wo[(16 * j + 8) * wpo + ko];
                const uint32_t a0 = wa & mask_a0, a2 = wa & mask_a2, a1 = wb & mask_a0, a3 = wb & mask_a2;
#pragma unroll
                for (int t = 0; t < NTS; ++t) {
                  const uint32_t b0 = FR ? fro[t][FR ? ko : 0][0] : qfr[((t * KK + wpt + ko) * 2 + 0) * 32];
                  const uint32_t b1 = FR ? fro[t][FR ? ko : 0][1] : qfr[((t * KK + wpt + ko) * 2 + 1) * 32];
                  mma_u8s8(ao[j][t], a0, a1, a2, a3, b0, b1);
                }
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < SU; ++j) {
          const int u = u0 + j;
          const __half2* nrm = reinterpret_cast<const __half2*>(stg + ST.knorm) + 16 * u;
          const float2 n_r = __half22float2(nrm[r]), n_r8 = __half22float2(nrm[r + 8]);
#pragma unroll
          for (int t = 0; t < NTS; ++t) {
            // each limb pair is exact in int32; the two pairs of a head meet across lanes q, q ^ 1
            float pi_r = static_cast<float>(ai[j][t][0] + 256 * ai[j][t][1]) * limb_w;
            float pi_r8 = static_cast<float>(ai[j][t][2] + 256 * ai[j][t][3]) * limb_w;
            float po_r = static_cast<float>(ao[j][t][0] + 256 * ao[j][t][1]) * limb_w;
            float po_r8 = static_cast<float>(ao[j][t][2] + 256 * ao[j][t][3]) * limb_w;
            pi_r += __shfl_xor_sync(0xffffffffu, pi_r, 1);
            pi_r8 += __shfl_xor_sync(0xffffffffu, pi_r8, 1);
            po_r += __shfl_xor_sync(0xffffffffu, po_r, 1);
            po_r8 += __shfl_xor_sync(0xffffffffu, po_r8, 1);
            // <sq, sign> = 2 * sum_{bit set} - sum_all, back to sq units by 2^-F in cin / cout
            const float s_r =
                cin[t] * n_r.x * fmaf(2.0f, pi_r, -xin[t]) + cout[t] * n_r.y * fmaf(2.0f, po_r, -xout[t]);
            const float s_r8 =
                cin[t] * n_r8.x * fmaf(2.0f, pi_r8, -xin[t]) + cout[t] * n_r8.y * fmaf(2.0f, po_r8, -xout[t]);
            const int hd = 2 * t + (q >> 1);
            if ((q & 1) == 0 && hd < G) {
              Sw[hd * kSStride + 16 * u + r] = s_r;
              Sw[hd * kSStride + 16 * u + r + 8] = s_r8;
            }
          }
        }
      }
      __syncwarp();
      // ---------------- online softmax, one lane per token (tokens lane, lane + 32)
      const bool v0 = lane < n_valid, v1 = lane + 32 < n_valid;
      float alpha[G];
      bool rescale = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float* srow = Sw + h * kSStride;
        const float s0 = srow[lane], s1 = srow[lane + 32];
        if (p.scores != nullptr) {
          float* gsc = p.scores + (static_cast<int64_t>(it.b) * p.Hq + it.hk * G + h) * p.T + tile0;
          if (v0) gsc[lane] = s0;
          if (v1) gsc[lane + 32] = s1;
        }
        // slots past the length may hold anything: they leave as -inf, p = 0
        const float l0 = v0 ? s0 * p.sm_scale_log2 : -INFINITY;
        const float l1 = v1 ? s1 * p.sm_scale_log2 : -INFINITY;
        float mx = fmaxf(l0, l1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float new_m = fmaxf(run_m[h], mx);  // finite: token 0 of the tile is valid
        alpha[h] = exp2f(run_m[h] - new_m);
        rescale |= alpha[h] != 1.0f;
        const float p0 = exp2f(l0 - new_m), p1 = exp2f(l1 - new_m);
        run_l[h] = fmaf(run_l[h], alpha[h], p0 + p1);
        run_m[h] = new_m;
        zacc[h] *= alpha[h];
        srow[lane] = p0;
        srow[lane + 32] = p1;
      }
      if (rescale) {  // warp-uniform
#pragma unroll
        for (int v = 0; v < NTV; ++v) {
          float a = 1.0f;
#pragma unroll
          for (int h = 0; h < G; ++h)
            if (h == 4 * v + q) a = alpha[h];
#pragma unroll
          for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int P = 0; P < 2; ++P)
#pragma unroll
              for (int k = 0; k < 4; ++k) vacc[g][P][v][k] *= a;
        }
      }
      __syncwarp();
      // ---------------- values: 4 steps of 16 tokens
      const uint32_t code_base = smem_u32(stg + ST.vcode);
      const uint32_t* szw = reinterpret_cast<const uint32_t*>(stg + ST.vsz);  // [64][4] (scale, zero) fp16 pairs
      const int mi = lane >> 3, mrow = lane & 7;
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {
        // codes first: they do not depend on the B operand built below
        // matrices: (group 2c, tokens 0-7), (2c, 8-15), (2c+1, 0-7), (2c+1, 8-15) of the 16
        uint32_t R[2][4];
#pragma unroll
        for (int call = 0; call < 2; ++call) {
          const int tok = 16 * u + 8 * (mi & 1) + mrow;
          const int grp = 2 * call + (mi >> 1);
          ldmatrix_x4_trans(R[call], code_base + tok * (kHeadDim / 2) + 16 * vcode_chunk(tok, grp));
        }
        {  // B operand: w = p * scale as fp16 hi + lo for tokens 16u + 2tp, +1 and group gq
          const int t0i = 16 * u + 2 * tp;
          const uint32_t sz0 = szw[t0i * 4 + gq], sz1 = szw[(t0i + 1) * 4 + gq];
          const bool ok0 = t0i < n_valid, ok1 = t0i + 1 < n_valid;
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&sz0));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&sz1));
          const float sc0 = ok0 ? f0.x : 0.0f, z0 = ok0 ? f0.y : 0.0f;
          const float sc1 = ok1 ? f1.x : 0.0f, z1 = ok1 ? f1.y : 0.0f;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float2 pp = *reinterpret_cast<const float2*>(Sw + h * kSStride + t0i);
            const float w0 = pp.x * sc0, w1 = pp.y * sc1;
            const __half2 hi = __floats2half2_rn(w0, w1);
            const float2 hf = __half22float2(hi);
            const __half2 lo = __floats2half2_rn(w0 - hf.x, w1 - hf.y);
            Ww[(2 * h) * kWStride + gq * 8 + tp] = *reinterpret_cast<const uint32_t*>(&hi);
            Ww[(2 * h + 1) * kWStride + gq * 8 + tp] = *reinterpret_cast<const uint32_t*>(&lo);
            zacc[h] = fmaf(pp.x, z0, fmaf(pp.y, z1, zacc[h]));
          }
        }
        __syncwarp();
#pragma unroll
        for (int call = 0; call < 2; ++call) {
#pragma unroll
          for (int gi = 0; gi < 2; ++gi) {
            const int g = 2 * call + gi;
            const uint32_t xl = R[call][2 * gi], xh = R[call][2 * gi + 1];
            const uint32_t xl8 = xl >> 8, xh8 = xh >> 8;
            // M-tile rows 0-7: dims 32g + 4r + 2P, rows 8-15: the next dim; k = the 16 tokens
            const uint32_t A0[4] = {nib_lo_h2(xl), nib_hi_h2(xl), nib_lo_h2(xh), nib_hi_h2(xh)};
            const uint32_t A1[4] = {nib_lo_h2(xl8), nib_hi_h2(xl8), nib_lo_h2(xh8), nib_hi_h2(xh8)};
#pragma unroll
            for (int v = 0; v < NTV; ++v) {
              const int hd = 4 * v + (r >> 1);  // column r: head 4v + r/2, limb r % 2
              const bool live = (G % 4 == 0) || hd < G;
              const uint32_t* wrow = Ww + (2 * min(hd, G - 1) + (r & 1)) * kWStride + g * 8;
              const uint32_t b0 = live ? wrow[q] : 0u, b1 = live ? wrow[q + 4] : 0u;
              mma_f16(vacc[g][0][v], A0, b0, b1);
              mma_f16(vacc[g][1][v], A1, b0, b1);
            }
          }
        }
        __syncwarp();  // Ww is rewritten by the next step
      }
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    gs_base += it.n_stage;
    gt_base += it.n_tile;
    if (!ok) atomicExch(flag, 1);
    if (!FR) {  // fragments were read from the query block until now
      __syncwarp();
      if (lane == 0) mbar_arrive(&qfree[qb]);
    }

    // ---- this warp's partial for the item into combine buffer cb
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) zacc[h] += __shfl_xor_sync(0xffffffffu, zacc[h], off);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) run_l[h] += __shfl_xor_sync(0xffffffffu, run_l[h], off);
    }
    if (ok && il >= NB && !mbar_wait(&cfree[cb], ((il / NB) - 1) & 1)) {
      ok = false;
      atomicExch(flag, 1);
    }
    float* cw = reinterpret_cast<float*>(smem + L.comb) + (cb * NC + warp) * G * kPartStride;  // [G][kPartStride]
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
      for (int P = 0; P < 2; ++P)
#pragma unroll
        for (int v = 0; v < NTV; ++v) {
          const int hd = 4 * v + q;
          if (hd < G) {
            const int d = 32 * g + 4 * r + 2 * P;
            cw[hd * kPartStride + d] = vacc[g][P][v][0] + vacc[g][P][v][1];
            cw[hd * kPartStride + d + 1] = vacc[g][P][v][2] + vacc[g][P][v][3];
          }
        }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (tp == 0) cw[h * kPartStride + kHeadDim + gq] = zacc[h];
      if (lane == 0) {
        cw[h * kPartStride + kHeadDim + 4] = run_m[h];
        cw[h * kPartStride + kHeadDim + 5] = run_l[h];
      }
    }
    __threadfence_block();
    __syncwarp();
    if (lane == 0) mbar_arrive(&cfull[cb]);  // the combiner takes it from here
  }
}

template <int G, int WPT_MAX, int WPO_MAX, bool EXACT>
cudaError_t launch_cfg(const DecodeParams& p0, cudaStream_t s) {
  constexpr int WPO_A = WPO_MAX > 0 ? WPO_MAX : 1;
  constexpr bool FR = Shape<G>::NTS * (WPT_MAX + WPO_A) * 2 <= Shape<G>::FRAG_BUDGET;
  DecodeParams p = p0;
  p.nstage = decode_nstage<G>(p.m, p.m_out);
  if (p.nstage < 2) return cudaErrorInvalidConfiguration;
  const Smem L(G, Shape<G>::NC, Shape<G>::NB, p.m, p.m_out, p.nstage);
  if (!L.aligned()) return cudaErrorInvalidConfiguration;
  const size_t smem = static_cast<size_t>(L.total);
  auto kern = decode_kernel<G, WPT_MAX, WPO_MAX, FR, EXACT>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int n_items = p.B * p.Hkv * p.splits;
  // persistent: one CTA per SM at most (the shared memory holds one)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(n_items < p.grid ? n_items : p.grid));
  cfg.blockDim = dim3(Shape<G>::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// Exact word counts for m in {128, 256, 512} with m_out = 64, else bounds.
template <int G>
cudaError_t launch_g(const DecodeParams& p, cudaStream_t s) {
  const int wpt = p.m / 32, wpo = p.m_out / 32;
  if (wpo == 2) {
    if (wpt == 4) return launch_cfg<G, 4, 2, true>(p, s);
    if (wpt == 8) return launch_cfg<G, 8, 2, true>(p, s);
    if (wpt == 16) return launch_cfg<G, 16, 2, true>(p, s);
  }
  if (wpo == 0) return launch_cfg<G, 16, 0, false>(p, s);
  return launch_cfg<G, 16, 8, false>(p, s);
}

}  // namespace

// A fragments of the query projection's bf16 m16n8k16 MMA: for 16-row tile
// mt of [S; S_out], 16-channel step ks and lane l = 4r + q, eight bf16 values
// (registers a0..a3, low half first): rows 16mt + r and 16mt + r + 8 at
// channels 16ks + 2q, +1 (a0, a1) and 16ks + 2q + 8, +9 (a2, a3).
void decode_fill_s_frag(const uint16_t* S, const uint16_t* S_out, int m, int m_out, uint16_t* out) {
  const int ksteps = kHeadDim / 16;
  for (int mt = 0; mt < (m + m_out) / 16; ++mt)
    for (int ks = 0; ks < ksteps; ++ks)
      for (int l = 0; l < 32; ++l) {
        const int r = l >> 2, q = l & 3;
        auto at = [&](int row, int c) {
          return row < m ? S[static_cast<size_t>(row) * kHeadDim + c] : S_out[static_cast<size_t>(row - m) * kHeadDim + c];
        };
        uint16_t* o = out + ((static_cast<size_t>(mt) * ksteps + ks) * 32 + l) * 8;
        const int r0 = 16 * mt + r, r1 = r0 + 8, c0 = 16 * ks + 2 * q;
        o[0] = at(r0, c0);
        o[1] = at(r0, c0 + 1);
        o[2] = at(r1, c0);
        o[3] = at(r1, c0 + 1);
        o[4] = at(r0, c0 + 8);
        o[5] = at(r0, c0 + 9);
        o[6] = at(r1, c0 + 8);
        o[7] = at(r1, c0 + 9);
      }
}

cudaError_t launch_decode(const DecodeParams& p0, qjl_dtype dt, cudaStream_t s) {
  DecodeParams p = p0;
  p.q_fp32 = dt == QJL_FP32 ? 1 : 0;
  switch (p.Hq / p.Hkv) {
    case 1: return launch_g<1>(p, s);
    case 2: return launch_g<2>(p, s);
    case 4: return launch_g<4>(p, s);
    case 8: return launch_g<8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qjl
