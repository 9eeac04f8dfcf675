// QJL decode attention, and the decode step that first appends one token.
//
// QJL summary (atlas.scime.ai), Approach: the query is JL-projected WITHOUT
// quantisation and a cached token's score is the unbiased asymmetric estimator
//   s_t = sqrt(pi/2)/m * |k_in| * <S q_in, sign(S k_in)>
//       + sqrt(pi/2)/m_out * |k_out| * <S_out q_out, sign(S_out k_out)>.
// With packed bits, <sq, sign> = 2 * sum_{bit set} sq_i - sum_i sq_i.
// p = online softmax of sm_scale * s; o = sum_t p_t (code_t * scale_t + zero_t).
// A decode step also sketches the key of each sequence's new token as it
// arrives (Approach: keys are quantised when they are generated, with no
// calibration) and quantises its value, in the same launch, and attends over
// it as well.
//
// Two launches per call, the second with a programmatic dependency on the
// first so that it starts while the first finishes.
//
// Prep kernel (decode_prep_kernel), one CTA of 10 warps per (sequence, kv head)
//    pair: builds the pair's query block in the workspace: the G = Hq/Hkv
//    queries of the pair projected on the tensor cores (sq = S q_in,
//    S_out q_out; bf16 operands, fp32 accumulation) and turned into integers
//    x_i = rint(sq_i * 2^F) with |x_i| < 2^29 (a power-of-two scale per head
//    and part), then x'_i = round(x_i / 2^(i mod 8)) so that the sign bit of
//    row i, which sits at bit (i mod 8) of its byte, enters the score MMA as
//    the byte value 2^(i mod 8) without a shift; x' is stored as four int8
//    limbs per entry in the per-lane B fragment order of the score MMA,
//    followed by F and sum_i 2^(i mod 8) x'_i. In a decode step it also
//    writes the pair's new token into its cache slot: the key's sign sketch
//    from the same tensor-core projection (a sign within a guard band of zero
//    is recomputed in fp64) with fp64 norms, and the value's codes. A
//    pair without tokens gets a zero output here.
//
// Decode kernel (decode_kernel), persistent, at most one CTA per SM; the CTAs
//    never wait for one another. The cache tiles of all pairs, in (sequence,
//    kv head, token) order, are cut into `grid` contiguous ranges of (almost)
//    equal length (stream-K); a CTA's range is a run of segments, each a tile
//    range of one pair.
//    * The producer warp streams the range into a shared-memory ring, several
//      consecutive tiles per cp.async.bulk copy (mbarrier completion, L2
//      evict-first policy, no multicast), and each segment's query block into
//      one of two buffers. It starts at once; the copies that depend on the
//      prep kernel (query blocks, the stage that holds an appended token) wait
//      for it.
//    * The consumer warps (14, or 6 at G = 8, so that the register file holds
//      all warps) take the tiles of a segment round-robin. Per tile:
//      - scores on the tensor cores: the A fragment of an int8 m16n8k32 MMA is
//        the sign word masked to one bit per byte (byte values 2^(i mod 8)); one
//        N-tile of 8 columns carries the 4 limbs of 2 heads; the limb sums are
//        exact in int32 and combined in fp32;
//      - online softmax per head over the tile with one lane per token (exp2
//        with log2(e) folded into the scale);
//      - values on the tensor cores, 16 tokens at a time: A = value codes of 16
//        dims of one group (ldmatrix.trans of the staged tile, each nibble
//        taken as an exact fp16 subnormal by one AND), B = p * scale split into fp16 hi and lo
//        columns (22 significant bits), fp32 accumulation; the zero-point term
//        sum_t p_t * zero_t is accumulated per group on CUDA cores.
//    * After a segment each consumer warp writes its partial (max, sum, o) to
//      shared memory; the combiner warp merges them and writes the output of a
//      pair the CTA holds whole, or else the segment's partial, and the last
//      CTA to finish a shared pair (an atomic ticket) merges its partials.
//      There is no CTA-wide barrier in the loop.
//    * Given ML (qjl_decode_attention_partial, one rank's shard of a
//      context-parallel decode), every output is left unnormalised and its
//      (max, sum) is written beside it, for qjl_merge_partials.
// Every wait (mbarrier, ring fill number) is bounded in time;
// on a timeout the kernel sets an error bit in the workspace header, writes NaN
// to the outputs it owns and returns.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

constexpr int kTT = kDecodeTileTokens;  // tokens per tile (the cache capacity is a multiple)
constexpr int kMaxStages = 8;           // ring stages of kStageTiles tiles (the count is set per launch)
constexpr int kNQ = kDecodeQBuffers;    // query-block buffers (by segment parity)
// per (warp, head) partial: o[d], zero sums[4], max, sum, padded to whole 16-byte
// vectors (the combiner reads o as float4)
constexpr int kPartStride = kHeadDim + 8;
static_assert(kPartStride % 4 == 0, "combine-buffer rows must stay 16-byte aligned");
constexpr int kSStride = 72;            // floats per head in a warp's score / probability buffer (padded)
constexpr int kWStride = 36;            // words per (head, limb) in a warp's value B-operand buffer (padded)
constexpr int kSmemBudget = 227 * 1024;
constexpr int kInfoWords = 4 + 32;  // partition info (long long): total tiles, b0, tiles before b0; scan scratch
constexpr uint64_t kDrainCycles = 4000000000ull;  // ~2 s: the limit of the wait for the copies in flight

// Launch shape by heads per kv head.
template <int G>
struct Shape {
  static constexpr int NC = G <= 4 ? 14 : 6;  // consumer warps
  static constexpr int THREADS = 32 * (NC + 2);  // + producer warp + combiner warp
  static constexpr int NTS = (G + 1) / 2;  // score N-tiles: 2 heads x 4 limbs
  static constexpr int NTV = (G + 3) / 4;  // value N-tiles: 4 heads x (hi, lo)
  static constexpr int NB = G <= 2 ? 2 : 1;  // combine buffers
  // query fragments held in registers when they fit this many (G = 4 reads them
  // from shared memory: the registers go to more consumer warps instead)
  static constexpr int FRAG_BUDGET = G <= 2 ? 24 : (G == 4 ? 0 : 96);
};
constexpr int kPrepWarps = 10;  // warps of a prep CTA (one query block and appended token each)

// ------------------------------------------------------------------ PTX helpers
// n / d and n % d by one multiply-high with m = ceil(2^32 / d) (division by an
// invariant integer through multiplication, Granlund and Montgomery 1994): the
// excess of m over 2^32 / d is below 1, so the quotient is exact for every
// 0 <= n < 2^32 / d, 2^29 for the ring's d <= 8 (a cache that fits in device
// memory has fewer than 2^24 ring stages: a stage is at least 14 KB).
struct DivMod {
  uint32_t d, m;
  __device__ __forceinline__ explicit DivMod(uint32_t d_) : d(d_), m(0xFFFFFFFFu / d_ + 1u) {}
  __device__ __forceinline__ int div(int n) const { return static_cast<int>(__umulhi(static_cast<uint32_t>(n), m)); }
  __device__ __forceinline__ int mod(int n, int q) const { return n - q * static_cast<int>(d); }
};
// 2^x by the hardware approximation, results below 2^-126 flushed to zero
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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
// Whether the phase with the given parity has completed; the thread waits at
// most about hint_ns for it before the call returns false.
// The wait limits below are counted in SM clock cycles (clock64: one-cycle
// resolution), `limit` = the context's limit in ns times the clock rate.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete; false after `limit`
// cycles (each try suspends at most about 1 us, or `limit` cycles if shorter).
// The first try is inline; only a wait that goes on calls out.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, uint64_t limit, uint32_t hint) {
  const uint64_t t0 = clock64();
  while (!mbar_try_wait_hint(bar, parity, hint)) {
    if (static_cast<uint64_t>(clock64()) - t0 > limit) return false;
  }
  return true;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const uint32_t hint = static_cast<uint32_t>(limit < 1000ull ? limit : 1000ull);
  if (mbar_try_wait_hint(bar, parity, hint)) return true;
  return mbar_wait_slow(bar, parity, limit, hint);
}
// Wait until a ring slot's published fill number reaches `fill`; false after
// `limit` cycles. The first check is inline; only a wait that goes on calls out.
__device__ __noinline__ bool seq_wait_slow(const int* seq, int fill, uint64_t limit) {
  const volatile int* v = seq;
  const uint64_t t0 = clock64();
  while (*v < fill) {
    __nanosleep(64);  // leave the issue slots to the other warps of the SM
    if (static_cast<uint64_t>(clock64()) - t0 > limit) return false;
  }
  __threadfence_block();
  return true;
}
__device__ __forceinline__ bool seq_wait(const int* seq, int fill, uint64_t limit) {
  if (*reinterpret_cast<const volatile int*>(seq) >= fill) {
    __threadfence_block();
    return true;
  }
  return seq_wait_slow(seq, fill, limit);
}
// Generic-proxy writes to global memory before this fence are seen by later
// bulk (async-proxy) copies.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
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
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint4& a, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(row_addr));
}
// Two fp16 values from the nibbles of a 32-bit word with one AND: a nibble n
// kept in bits 0-3 (or 4-7) of a 16-bit half, the exponent field zero, is the
// exact fp16 subnormal n * 2^-24 (or n * 2^-20). The value MMA takes the codes
// in that form; its sums are scaled back by 2^24 (2^20) when a partial is
// written.
__device__ __forceinline__ uint32_t nib_lo_h2(uint32_t x) { return x & 0x000F000Fu; }
__device__ __forceinline__ uint32_t nib_hi_h2(uint32_t x) { return x & 0x00F000F0u; }
constexpr float kNibLoScale = 16777216.0f;  // 2^24
constexpr float kNibHiScale = 1048576.0f;   // 2^20

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

// Named barrier `id` (1 .. 3; 0 is __syncthreads) over `threads` threads.
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}


// ------------------------------------------------------------------ layouts
// A ring stage holds kStageTiles consecutive cache tiles exactly as they lie in
// global memory (TileLayout offsets inside each tile).
struct Smem {
  // byte offsets from the dynamic shared-memory base
  int stages, bars, qbuf, comb, sbuf, wbuf, info, misc, total, qblock;
  __host__ __device__ Smem(int G, int NC, int NB, int m, int m_out, int nstage, int vbits) {
    const TileLayout tl = tile_layout(m, m_out, vbits);
    qblock = static_cast<int>(decode_qblock_bytes(G, m, m_out));
    stages = 0;
    // full, empty [kMaxStages]; qfull, qfree [kNQ]; cfree, cfull [2]
    bars = stages + nstage * kStageTiles * tl.bytes;
    qbuf = bars + (2 * kMaxStages + 2 * kNQ + 4) * 8;  // query blocks [kNQ] (bulk-copy targets)
    comb = qbuf + kNQ * qblock;                        // fp32 [NB][NC][G][kPartStride]
    sbuf = comb + NB * NC * G * kPartStride * 4;       // fp32 [NC][G][kSStride]
    wbuf = sbuf + NC * G * kSStride * 4;               // u32 [NC][2G][kWStride]
    info = wbuf + NC * 2 * G * kWStride * 4;           // long long [kInfoWords]
    misc = info + kInfoWords * 8;                      // fill sequence [kMaxStages], flags
    total = misc + (kMaxStages + 4) * 4;
  }
  // every section starts on a 16-byte boundary (bulk copies, vector accesses)
  __host__ __device__ bool aligned() const {
    return ((stages | bars | qbuf | comb | sbuf | wbuf | info | misc | qblock) & 15) == 0;
  }
};
// Ring stages that fit the shared-memory budget (at most kMaxStages, 0 if not even 2 fit).
template <int G>
int decode_nstage(int m, int m_out, int vbits) {
  for (int n = kMaxStages; n >= 2; --n)
    if (Smem(G, Shape<G>::NC, Shape<G>::NB, m, m_out, n, vbits).total <= kSmemBudget) return n;
  return 0;
}

// ------------------------------------------------------------------ partition
// Tokens of sequence b that this call attends over (its length, plus the
// appended token in a decode step), and their 64-token tiles.
__device__ __forceinline__ int seq_len(const DecodeParams& p, int b) {
  int len = p.seqlens ? p.seqlens[b] : p.T;
  len = max(0, min(len, p.T));
  return len + p.append;
}
__device__ __forceinline__ int seq_tiles(const DecodeParams& p, int b) { return (seq_len(p, b) + kTT - 1) / kTT; }

// Stream-K partition of the flattened (sequence, kv head, tile) sequence:
// CTA c holds tiles [start(c), start(c + 1)), start(c) = floor(total c / grid),
// evaluated as q c + floor(rem c / grid) (total = q grid + rem) so that only
// the set-up divides 64-bit numbers.
struct Part {
  long long total, q;
  int grid, rem;
  __device__ Part(long long total_, int grid_) : total(total_), q(total_ / grid_), grid(grid_),
                                                 rem(static_cast<int>(total_ - total_ / grid_ * grid_)) {}
  __device__ long long start(int c) const { return q * c + (rem * c) / grid; }
  __device__ bool empty(int c) const { return start(c) == start(c + 1); }
  // the CTA whose range holds tile x (x < total): the largest c with start(c) <= x
  __device__ int owner(long long x) const {
    int c = min(grid - 1, static_cast<int>(static_cast<double>(x) * grid / static_cast<double>(total)));
    while (c + 1 < grid && start(c + 1) <= x) ++c;
    while (c > 0 && start(c) > x) --c;
    return c;
  }
};

// One segment: tiles [lo, hi) of pair bh (sequence b, kv head hk), whose first
// tile is tile `first` of the flattened sequence; il = its place in the CTA's run.
struct Seg {
  int b, hk, lo, hi, nt, len, il;
  long long bh, first;
  __device__ int t0() const { return lo * kTT; }
  __device__ int t1() const { return min(hi * kTT, len); }
  __device__ int n_tile() const { return hi - lo; }
  __device__ int n_stage() const { return (hi - lo + kStageTiles - 1) / kStageTiles; }
  __device__ bool whole() const { return lo == 0 && hi == nt; }
};
// Walks the segments of a CTA's range in order (every role walks the same list).
struct SegIter {
  int b;
  long long cum;  // tiles of the sequences before b
  long long x, x_end;
  int il;
  __device__ bool next(const DecodeParams& p, Seg& s) {
    if (x >= x_end) return false;
    int nt = seq_tiles(p, b);
    while (x >= cum + static_cast<long long>(p.Hkv) * nt) {  // sequences without tiles take no room
      cum += static_cast<long long>(p.Hkv) * nt;
      ++b;
      nt = seq_tiles(p, b);
    }
    const int hk = static_cast<int>((x - cum) / nt);
    s.b = b;
    s.hk = hk;
    s.bh = static_cast<long long>(b) * p.Hkv + hk;
    s.nt = nt;
    s.len = seq_len(p, b);
    s.first = cum + static_cast<long long>(hk) * nt;
    s.lo = static_cast<int>(x - s.first);
    s.hi = static_cast<int>(min(static_cast<long long>(nt), x_end - s.first));
    s.il = il++;
    x = s.first + s.hi;
    return true;
  }
};

// The total tile count and, for the first tile x0 of this CTA's range, the
// sequence b0 that holds it and the tiles before b0 (prefix sums of the tile
// counts over the sequences; all threads of the CTA take part, the caller
// synchronises). info[0] = total, info[1] = b0, info[2] = tiles before b0.
template <int THREADS>
__device__ void locate(const DecodeParams& p, long long* info) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = THREADS / 32;
  long long* scan = info + 4;
  if (p.seqlens == nullptr) {  // every sequence has the same length
    if (threadIdx.x == 0) {
      const long long per_b = static_cast<long long>(p.Hkv) * seq_tiles(p, 0);
      const long long total = per_b * p.B;
      const long long x0 = total * blockIdx.x / gridDim.x;
      const long long b0 = per_b > 0 ? x0 / per_b : p.B;
      info[0] = total;
      info[1] = b0;
      info[2] = b0 * per_b;
    }
    return;
  }
  const int chunk = (p.B + THREADS - 1) / THREADS;
  const int lo = min(p.B, static_cast<int>(threadIdx.x) * chunk), hi = min(p.B, lo + chunk);
  long long s = 0;
  for (int b = lo; b < hi; ++b) s += seq_tiles(p, b);
  s *= p.Hkv;
  long long v = s;  // inclusive scan over the CTA
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  if (lane == 31) scan[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < NW ? scan[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    if (lane < NW) scan[lane] = w;
  }
  __syncthreads();
  const long long incl = v + (warp > 0 ? scan[warp - 1] : 0), excl = incl - s;
  const long long total = scan[NW - 1];
  const long long x0 = total * blockIdx.x / gridDim.x;
  if (threadIdx.x == 0) info[0] = total;
  if (x0 >= total) {
    if (threadIdx.x == 0) {
      info[1] = p.B;
      info[2] = total;
    }
  } else if (excl <= x0 && x0 < incl) {  // exactly one thread: the one whose sequences hold tile x0
    long long c = excl;
    int b = lo;
    for (; b < hi; ++b) {
      const long long t = static_cast<long long>(p.Hkv) * seq_tiles(p, b);
      if (x0 < c + t) break;
      c += t;
    }
    info[1] = b;
    info[2] = c;
  }
}

// ------------------------------------------------------------------ query blocks
// Query block of one (b, kv head) (bytes), built by the prep kernel in the workspace:
//   fragment word h of lane l for N-tile t and word kk at word index ((kk * 32 + l) * NTS + t) * 2 + h
//   (a lane's N-tiles side by side: one 16-byte load for two of them):
//   for lane (r, q) (column r of N-tile t: head 2t + r/4, limb r % 4), byte j
//   holds that limb of x'[head] at sketch row 32kk + 2q + h + 8j (kk < m/32:
//   inlier rows, then outlier rows); then int32 F[G][2] and int64 sum[G][2]
//   (inlier, outlier part).

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

// This lane's B-fragment channels 16 ks + 2q + (e & 1) + 8 (e >> 1), e = 0..3.
__device__ __forceinline__ int frag_channel(int ks, int q, int e) { return 16 * ks + 2 * q + (e & 1) + 8 * (e >> 1); }

// The outlier channels of a pair as a 128-bit mask (lane o < n_out holds channel c_idx, else -1).
__device__ __forceinline__ void outlier_mask(int c_idx, uint32_t (&om)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k)
    om[k] = __reduce_or_sync(0xffffffffu, c_idx >= 0 && (c_idx >> 5) == k ? 1u << (c_idx & 31) : 0u);
}
__device__ __forceinline__ bool is_outlier(const uint32_t (&om)[4], int c) { return ((om[c >> 5] >> (c & 31)) & 1u) != 0u; }

// One bf16 B fragment pair (channels 2q, 2q+1 and 2q+8, 2q+9 of a 16-channel
// step) as up to three bf16 limbs whose sum is exact: an fp32 value has 24
// significant bits, each bf16 rounding keeps 8 and the remainder is exact in
// fp32, so after two limbs at most 8 bits are left for the third.
__device__ __forceinline__ void bf16_limbs(const float (&v)[4], uint32_t (&lb)[3][2]) {
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
}

// The global loads of a build, issued ahead of it: this lane's query values
// (head r, channels frag_channel(ks, q, e)) and one outlier index per lane.
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

// One query-block build: the query block of a pair into dst (global memory),
// run by the nw warps wi = 0 .. nw-1 (one named barrier `bar` inside, over
// those warps); the caller then runs build_finish after a barrier over the
// same warps. sums and maxes (shared memory, per (head, part)) start at zero.
// Sketch row i (inlier rows 0 .. m-1, then outlier rows) is the dot product of
// row i of S (or of S_out) with the query restricted to the inlier (or to the
// outlier) channels, on the tensor cores: sq[rows x G] = S[rows x d] q[d x G]
// as bf16 m16n8k16 MMAs with fp32 accumulation; the A fragments come from
// S_frag (L2-resident), the B fragments are the query (an fp32 query as three
// exact bf16 limbs, each its own MMA).
// Warp wi takes the 32-row words kk = wi, wi + nw, ...: the two 16-row tiles
// of a word, kept in registers while the warps exchange their maxima (F per
// (head, part) from max|sq|), then x = rint(sq 2^F) (an exact scaling) and
// x' = round(x / 2^(i mod 8)) in the accumulator lanes, moved into the
// fragment lanes by shuffles and packed as int8 limbs; the word's sums of
// 2^(i mod 8) x'_i are added to sums[head][part] (shared atomics).
template <int G, int WMAX>
__device__ __forceinline__ void build_qblock(const DecodeParams& p, const QLoad& ql, unsigned char* dst,
                                             unsigned long long* sums, unsigned int* maxes, int wi, int nw, int bar) {
  constexpr int NTS = (G + 1) / 2;
  constexpr int KS = kHeadDim / 16;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2, q = lane & 3;
  const int m = p.m, m_out = p.m_out;
  const int wpt = m >> 5, wpo = m_out >> 5, KK = wpt + wpo;

  const float (&qv)[KS][4] = ql.qv;
  uint32_t om[4];
  outlier_mask(ql.c_idx, om);
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
      for (int e = 0; e < 4; ++e) v[e] = is_outlier(om, frag_channel(ks, q, e)) == (part == 1) ? qv[ks][e] : 0.0f;
      uint32_t lb[3][2];
      bf16_limbs(v, lb);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint4 a = __ldg(p.S_frag + (static_cast<int64_t>(mt + u) * KS + ks) * 32 + lane);
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
  named_sync(bar, 32 * nw);
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
        fr[((kk * 32 + lane) * NTS + t) * 2 + h] = head < G ? v : 0u;
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

// ------------------------------------------------------------------ the appended token
// Element c of the appended key / value row of pair (b, hk).
__device__ __forceinline__ float kv_elem(const DecodeParams& p, const void* base, int64_t off, int c) {
  return p.q_fp32 ? static_cast<const float*>(base)[off + c]
                  : __bfloat162float(static_cast<const __nv_bfloat16*>(base)[off + c]);
}

// The sign of S_i k_in (part 0) or S_out,i k_out (part 1) from the exact
// products summed in fp64, for a projection within the guard band of zero; the
// whole warp takes part (lane l: channels 4l .. 4l+3), the result is uniform.
__device__ __noinline__ bool exact_sign(const DecodeParams& p, int part, int i, int64_t koff, uint32_t om0,
                                        uint32_t om1, uint32_t om2, uint32_t om3) {
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* row = (part ? p.S_out : p.S) + static_cast<int64_t>(i) * kHeadDim;
  const uint32_t om = lane < 8 ? om0 : (lane < 16 ? om1 : (lane < 24 ? om2 : om3));  // bits of channels 32k..32k+31
  double y = 0.0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = 4 * lane + e;
    if (((om >> (c & 31)) & 1u) != static_cast<uint32_t>(part)) continue;
    y = fma(static_cast<double>(__bfloat162float(row[c])), static_cast<double>(kv_elem(p, p.K_new, koff, c)), y);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
  return y >= 0.0;
}

// The sign sketch of pair bh's new key into cache slot `pos`, by the nw warps
// wi = 0 .. nw-1 (no barrier inside): warp wi takes the 32-row words
// kk = wi, wi + nw, ... The projections run on the tensor cores as in
// build_qblock, with the key as the only B column; a projection whose
// magnitude is below p.guard times the norm of its part (far above the fp32
// rounding of the sums) is recomputed in fp64 from the exact products, so the
// bit is the sign of the exact projection. Norms are summed in fp64 and stored
// as fp16, as in qjl_quantize_keys.
template <int WMAX>
__device__ __forceinline__ void append_key(const DecodeParams& p, int b, int hk, int64_t bh, int pos, int c_idx,
                                           int wi, int nw) {
  constexpr int KS = kHeadDim / 16;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2, q = lane & 3;
  const int m = p.m, m_out = p.m_out;
  const int wpt = m >> 5, wpo = m_out >> 5, KK = wpt + wpo;
  const int64_t koff = static_cast<int64_t>(b) * p.k_sb + static_cast<int64_t>(hk) * p.k_sh;
  uint32_t om[4];
  outlier_mask(c_idx, om);
  // norms of the inlier and outlier parts in fp64 (lane l: channels 4l .. 4l+3)
  double n2_in = 0.0, n2_out = 0.0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c = 4 * lane + e;
    const double x = kv_elem(p, p.K_new, koff, c);
    if (is_outlier(om, c))
      n2_out = fma(x, x, n2_out);
    else
      n2_in = fma(x, x, n2_in);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    n2_in += __shfl_xor_sync(0xffffffffu, n2_in, off);
    n2_out += __shfl_xor_sync(0xffffffffu, n2_out, off);
  }
  const double norm_in = sqrt(n2_in), norm_out = sqrt(n2_out);
  int j;
  unsigned char* tile = tile_of(p.tiles, p.tl, bh, p.cap, pos, &j);
  if (wi == 0 && lane == 0) {
    __half* kn = reinterpret_cast<__half*>(tile + p.tl.knorm) + 2 * j;
    kn[0] = __double2half(norm_in);
    kn[1] = __double2half(norm_out);
  }
  // B column 0 = the key (lanes with r == 0), the other columns zero
  float kv[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks)
#pragma unroll
    for (int e = 0; e < 4; ++e) kv[ks][e] = r == 0 ? kv_elem(p, p.K_new, koff, frag_channel(ks, q, e)) : 0.0f;
#pragma unroll
  for (int w = 0; w < WMAX; ++w) {
    const int kk = wi + w * nw;
    if (kk >= KK) break;
    const int part = kk < wpt ? 0 : 1;
    const int mt = part ? (m + 32 * (kk - wpt)) / 16 : 2 * kk;
    float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = is_outlier(om, frag_channel(ks, q, e)) == (part == 1) ? kv[ks][e] : 0.0f;
      uint32_t lb[3][2];
      bf16_limbs(v, lb);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint4 a = __ldg(p.S_frag + (static_cast<int64_t>(mt + u) * KS + ks) * 32 + lane);
        mma_bf16(acc[u], a, lb[0][0], lb[0][1]);
        if (p.q_fp32) {
          mma_bf16(acc[u], a, lb[1][0], lb[1][1]);
          mma_bf16(acc[u], a, lb[2][0], lb[2][1]);
        }
      }
    }
    // column 0 sits in the lanes with q == 0: rows r (acc[u][0]) and r + 8 (acc[u][2]) of tile u
    uint32_t bits = 0u, near = 0u;
    if (q == 0) {
      const float thr = p.guard * static_cast<float>(part ? norm_out : norm_in);
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int row = 16 * u + 8 * hf + r;  // bit of the word
          const float y = acc[u][2 * hf];
          bits |= static_cast<uint32_t>(y >= 0.0f) << row;
          near |= static_cast<uint32_t>(fabsf(y) < thr) << row;
        }
    }
    uint32_t word = __reduce_or_sync(0xffffffffu, bits);
    // projections within the guard band: the sign of the exact sum, one row at a time
    for (uint32_t nb = __reduce_or_sync(0xffffffffu, near); nb != 0u; nb &= nb - 1u) {
      const int row = __ffs(static_cast<int>(nb)) - 1;
      const bool bit = exact_sign(p, part, 32 * (part ? kk - wpt : kk) + row, koff, om[0], om[1], om[2], om[3]);
      word = bit ? (word | (1u << row)) : (word & ~(1u << row));
    }
    if (lane == 0) {
      if (part)
        reinterpret_cast<uint32_t*>(tile + p.tl.kbits_out)[j * wpo + (kk - wpt)] = word;
      else
        reinterpret_cast<uint32_t*>(tile + p.tl.kbits)[j * wpt + kk] = word;
    }
  }
}

// The 4-bit codes of pair bh's new value into cache slot `pos`, by one warp:
// lane l quantises channels 4l .. 4l+3; the 8 lanes of a group of 32 dims
// share its min and max. Every step is the IEEE fp32 operation of
// qjl_quantize_values (zero = fp16(min), scale = fp16((max - min) / 15),
// code = clamp(rint((v - zero) / scale), 0, 15), code 0 when scale == 0).
__device__ __forceinline__ void append_value(const DecodeParams& p, int b, int hk, int64_t bh, int pos) {
  const int lane = threadIdx.x & 31;
  const int64_t voff = static_cast<int64_t>(b) * p.v_sb + static_cast<int64_t>(hk) * p.v_sh;
  float v[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] = kv_elem(p, p.V_new, voff, 4 * lane + e);
  float lo = fminf(fminf(v[0], v[1]), fminf(v[2], v[3])), hi = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  const int vb = p.tl.vbits, top = (1 << vb) - 1;
  const __half zero_h = __float2half_rn(lo);
  const __half scale_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), static_cast<float>(top)));
  const float zero = __half2float(zero_h), scale = __half2float(scale_h);
  uint32_t bits = 0u;
  if (scale != 0.0f) {
    const float rcp = __frcp_rn(scale);
#pragma unroll
    for (int e = 0; e < 4; ++e) bits |= value_code(v[e], zero, scale, rcp, top) << (vb * e);
  }
  int j;
  unsigned char* tile = tile_of(p.tiles, p.tl, bh, p.cap, pos, &j);
  const int g = lane >> 3;
  if (vb == 2) {  // dims 4l' .. 4l'+3 of group g (l' = lane % 8): the token's byte in line (g, l')
    tile[p.tl.vcode + v2_line(g, lane & 7) + j] = static_cast<unsigned char>(bits);
  } else {  // dims 4l' .. 4l'+3 of group g are bytes 2l', 2l'+1 of the group's 16 bytes
    reinterpret_cast<uint16_t*>(tile + p.tl.vcode + j * (kHeadDim / 2) + 16 * vcode_chunk(j, g))[lane & 7] =
        static_cast<uint16_t>(bits);
  }
  if ((lane & 7) == 0) {
    const uint32_t sz = static_cast<uint32_t>(__half_as_ushort(scale_h)) |
                        (static_cast<uint32_t>(__half_as_ushort(zero_h)) << 16);
    reinterpret_cast<uint32_t*>(tile + p.tl.vsz + j * (kHeadDim / kValueGroup) * 4)[g] = sz;
  }
}

// ------------------------------------------------------------------ prep kernel
// One CTA per (sequence, kv head) pair: its query block into the workspace
// and, in a decode step, its new token into the cache; a pair without tokens
// gets a zero output. The decode kernel launched next may start at once
// (launch_dependents) and waits for this grid before it reads what it wrote.
template <int G, int WMAX>
__global__ void __launch_bounds__(kPrepWarps * 32, 2) decode_prep_kernel(DecodeParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ unsigned long long sums[2 * G];  // per (head, part): sum of 2^(i mod 8) x'_i
  __shared__ unsigned int maxes[2 * G];       // per (head, part): max |sq| (float bits)
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x < 2 * G) {
    sums[threadIdx.x] = 0ull;
    maxes[threadIdx.x] = 0u;
  }
  __syncthreads();
  const int64_t bh = blockIdx.x;
  const int b = static_cast<int>(bh / p.Hkv), hk = static_cast<int>(bh % p.Hkv);
  const int len = seq_len(p, b);
  if (len == 0) {  // no tiles: the output of the pair is zero (as a part: max -inf, sum 0)
    for (int e = threadIdx.x; e < G * kHeadDim; e += blockDim.x)
      p.O[(static_cast<int64_t>(b) * p.Hq + hk * G) * kHeadDim + e] = 0.0f;
    if (p.ML && threadIdx.x < G) {
      const int64_t orow = static_cast<int64_t>(b) * p.Hq + hk * G + threadIdx.x;
      p.ML[2 * orow] = -INFINITY;
      p.ML[2 * orow + 1] = 0.0f;
    }
    return;
  }
  QLoad ql;
  load_query<G>(p, bh, ql);
  unsigned char* dst = p.qblock + bh * p.qblock_bytes;
  build_qblock<G, WMAX>(p, ql, dst, sums, maxes, warp, kPrepWarps, 1);
  __syncthreads();
  if (warp == kPrepWarps - 1) build_finish<G>(p, dst, sums, maxes);
  if (p.append) {
    append_key<WMAX>(p, b, hk, bh, len - 1, ql.c_idx, warp, kPrepWarps);
    if (warp == 0) append_value(p, b, hk, bh, len - 1);
  }
}

// ------------------------------------------------------------------ main kernel
// WPT_MAX / WPO_MAX bound the inlier / outlier sign words per token; with
// EXACT they are the exact counts, so that every word loop is fully static.
// VB: value code bits (4, or 2 for the line layout of 2-bit codes).
template <int G, int WPT_MAX, int WPO_MAX, bool FR, bool EXACT, int VB>
__global__ void __launch_bounds__(Shape<G>::THREADS, 1) decode_kernel(DecodeParams p) {
  constexpr int NC = Shape<G>::NC, NTS = Shape<G>::NTS, NTV = Shape<G>::NTV, NB = Shape<G>::NB;
  constexpr int THREADS = Shape<G>::THREADS;
  constexpr int WPO_A = WPO_MAX > 0 ? WPO_MAX : 1;
  constexpr int FRI = FR ? WPT_MAX : 1, FRO = FR ? WPO_A : 1;  // query fragments held in registers
  constexpr int SU = 1;  // score sub-tiles per pass (2 measured no faster and costs registers)
  extern __shared__ __align__(128) unsigned char smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = EXACT ? 32 * WPT_MAX : p.m, m_out = EXACT ? 32 * WPO_MAX : p.m_out;
  const int wpt = m >> 5, wpo = m_out >> 5, KK = wpt + wpo;
  const int nstage = p.nstage;
  const DivMod by_nstage(static_cast<uint32_t>(nstage));
  const uint64_t lim = p.wait_cycles;
  const Smem L(G, NC, NB, m, m_out, nstage, p.tl.vbits);
  const TileLayout ST = p.tl;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kMaxStages;
  uint64_t* qfull = empty + kMaxStages;
  uint64_t* qfree = qfull + kNQ;
  uint64_t* cfree = qfree + kNQ;
  uint64_t* cfull = cfree + 2;
  long long* info = reinterpret_cast<long long*>(smem + L.info);
  int* fill_seq = reinterpret_cast<int*>(smem + L.misc);  // [kMaxStages]: fill last issued into each ring slot
  int* flag = fill_seq + kMaxStages;                      // error flag

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstage; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kStageTiles);  // one arrival per tile (the producer stands in for missing tiles)
      fill_seq[s] = -1;
    }
    for (int k = 0; k < kNQ; ++k) {
      mbar_init(&qfull[k], 1);   // the producer's copy of the segment's query block
      mbar_init(&qfree[k], NC);  // every consumer warp releases every query block
    }
    for (int k = 0; k < NB; ++k) {
      mbar_init(&cfree[k], 1);   // the combiner releases the combine buffer
      mbar_init(&cfull[k], NC);  // every consumer warp posts its partial
    }
    *flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  locate<THREADS>(p, info);
  __syncthreads();
  const Part P(info[0], static_cast<int>(gridDim.x));
  SegIter seg0;  // this CTA's segments
  seg0.b = static_cast<int>(info[1]);
  seg0.cum = info[2];
  seg0.x = P.start(blockIdx.x);
  seg0.x_end = P.start(blockIdx.x + 1);
  seg0.il = 0;

  if (warp == NC) {
    // ============================================================ producer
    // (one lane: a blocking mbarrier wait stalls its whole warp, so no other
    // role shares this warp)
    if (lane == 0) {
      bool ok = true, prep_done = false;
      int pend = 0;  // segments 0 and 1 whose query-block copy waits for the prep kernel
      long long pend_bh0 = 0, pend_bh1 = 0;
      int last_q[2] = {-1, -1};  // the last segment whose query block was copied into each buffer
      const uint64_t stream_policy = evict_first_policy();
      const int64_t tiles_per_slab = p.cap / kTT;
      auto issue_q = [&](int il, long long bh) {
        const int kb = il % kNQ;
        mbar_arrive_expect_tx(&qfull[kb], L.qblock);
        bulk_g2s(smem + L.qbuf + kb * L.qblock, p.qblock + bh * p.qblock_bytes, L.qblock, &qfull[kb]);
        last_q[kb] = il;
      };
      // The query blocks and the appended tokens are written by the prep
      // kernel launched just before this one (a programmatic dependency: this
      // grid may start before the prep grid ends). Wait for it only when a
      // copy needs its results or there is nothing else to do.
      auto await_prep = [&]() {
        if (prep_done) return;
        asm volatile("griddepcontrol.wait;" ::: "memory");
        fence_proxy_async_global();
        prep_done = true;
        if (pend & 1) issue_q(0, pend_bh0);
        if (pend & 2) issue_q(1, pend_bh1);
        pend = 0;
      };
      SegIter it = seg0;
      Seg s;
      int gs = 0;  // stages issued so far (ring slot gs mod nstage, fill gs / nstage)
      while (ok && it.next(p, s)) {
        const int kb = s.il % kNQ;
        if (s.il >= kNQ) {
          await_prep();
          if (!mbar_wait(&qfree[kb], ((s.il / kNQ) - 1) & 1, lim)) {
            ok = false;
            break;
          }
          issue_q(s.il, s.bh);
        } else if (prep_done) {
          issue_q(s.il, s.bh);
        } else {
          pend |= 1 << s.il;
          if (s.il == 0)
            pend_bh0 = s.bh;
          else
            pend_bh1 = s.bh;
        }
        // the segment's tiles are consecutive in global memory
        const unsigned char* g_tile = p.tiles + (s.bh * tiles_per_slab + s.lo) * static_cast<int64_t>(ST.bytes);
        const int n_tile = s.n_tile(), n_stage = s.n_stage();
        for (int st = 0; st < n_stage && ok; ++st) {
          const int fill = by_nstage.div(gs), slot = by_nstage.mod(gs, fill);
          if (gs >= nstage) {
            await_prep();  // the ring is full: the consumers need their query blocks to go on
            if (!mbar_wait(&empty[slot], (fill - 1) & 1, lim)) {
              ok = false;
              break;
            }
          }
          // the stage that holds the token the prep kernel appended (the pair's last tile)
          if (p.append && s.hi == s.nt && st == n_stage - 1) await_prep();
          // Consumers skip stages that other warps consume, so a parity wait alone
          // could match an older phase: they first wait for this fill number.
          __threadfence_block();
          *reinterpret_cast<volatile int*>(&fill_seq[slot]) = fill;
          const int nt = min(kStageTiles, n_tile - st * kStageTiles);
          const uint32_t bytes = static_cast<uint32_t>(nt * ST.bytes);
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_g2s_hint(smem + L.stages + slot * kStageTiles * ST.bytes,
                        g_tile + static_cast<int64_t>(st) * kStageTiles * ST.bytes, bytes, &full[slot],
                        stream_policy);
          // a short stage: arrive for the tiles no consumer will release
          if (nt < kStageTiles) mbar_arrive_cnt(&empty[slot], kStageTiles - nt);
          ++gs;
        }
      }
      if (pend) await_prep();  // query blocks still to copy
      // Drain: every copy issued here lands before the CTA may exit (a query
      // block is copied only once the consumers released the block two
      // segments back, so only the last one per buffer can be in flight).
      // A copy lands within microseconds, so this wait is allowed kDrainCycles
      // even when the context's limit is shorter.
      const uint64_t drain = lim > kDrainCycles ? lim : kDrainCycles;
      for (int g = gs > nstage ? gs - nstage : 0; g < gs; ++g)
        if (!mbar_wait(&full[g % nstage], (g / nstage) & 1, drain)) ok = false;
      for (int kb = 0; kb < kNQ; ++kb)
        if (last_q[kb] >= 0 && !mbar_wait(&qfull[kb], (last_q[kb] / kNQ) & 1, drain)) ok = false;
      if (!ok) {
        atomicExch(flag, 1);
        atomicOr(p.hdr + 2, kDecodeErrTimeout);
      }
    }
  } else if (warp == NC + 1) {
    // ============================================================ combiner
    // Merges the consumer warps' partials of each segment, off the consumers'
    // critical path, and merges the partials of a pair split between CTAs.
    bool failed = false;
    SegIter it = seg0;
    Seg s;
    while (it.next(p, s)) {
      const int cb = s.il % NB;
      if (!failed && !mbar_wait(&cfull[cb], (s.il / NB) & 1, lim)) {
        failed = true;
        atomicExch(flag, 1);
        atomicOr(p.hdr + 2, kDecodeErrTimeout);
      }
      __threadfence_block();
      failed |= *reinterpret_cast<volatile int*>(flag) != 0;
      const float* cbuf = reinterpret_cast<const float*>(smem + L.comb) + cb * NC * G * kPartStride;
      const int hq0 = s.hk * G;
      const bool whole = s.whole();
      const int slot = s.il == 0 ? 2 * static_cast<int>(blockIdx.x) : 2 * static_cast<int>(blockIdx.x) + 1;
      // per head: the warps' maximum and weights once, then channels 4 lane .. 4 lane + 3
      for (int j = 0; j < G; ++j) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NC; ++w) M = fmaxf(M, cbuf[(w * G + j) * kPartStride + kHeadDim + 4]);
        float Lsum = 0.0f;
        float4 ov = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < NC; ++w) {
            const float* pw = cbuf + (w * G + j) * kPartStride;
            const float mw = pw[kHeadDim + 4];
            const float f = mw == -INFINITY ? 0.0f : exp2f(mw - M);
            Lsum = fmaf(pw[kHeadDim + 5], f, Lsum);
            const float4 o4 = reinterpret_cast<const float4*>(pw)[lane];
            const float z = pw[kHeadDim + (lane >> 3)];  // zero-point term of group (4 lane) / 32
            ov.x = fmaf(o4.x + z, f, ov.x);
            ov.y = fmaf(o4.y + z, f, ov.y);
            ov.z = fmaf(o4.z + z, f, ov.z);
            ov.w = fmaf(o4.w + z, f, ov.w);
          }
        }
        const int64_t orow = static_cast<int64_t>(s.b) * p.Hq + hq0 + j;
        const float nanv = __int_as_float(0x7fc00000);  // NaN marks a timed-out wait
        if (whole) {
          // normalised, or as a part (unnormalised, with its maximum and sum)
          const float inv = p.ML ? 1.0f : (Lsum > 0.0f ? 1.0f / Lsum : 0.0f);
          const float4 o = failed ? make_float4(nanv, nanv, nanv, nanv)
                                  : make_float4(ov.x * inv, ov.y * inv, ov.z * inv, ov.w * inv);
          reinterpret_cast<float4*>(p.O + orow * kHeadDim)[lane] = o;
          if (p.ML && lane == 0) {
            p.ML[2 * orow] = M;
            p.ML[2 * orow + 1] = Lsum;
          }
        } else {
          const int64_t prow = static_cast<int64_t>(slot) * G + j;
          reinterpret_cast<float4*>(p.part_o + prow * kHeadDim)[lane] = failed ? make_float4(nanv, nanv, nanv, nanv) : ov;
          if (lane == 0) {
            p.part_ml[2 * prow] = M;
            p.part_ml[2 * prow + 1] = Lsum;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cfree[cb]);
      if (!whole) {
        // ---- the last CTA to finish its part of this pair merges the parts
        const int c1 = P.owner(s.first), c2 = P.owner(s.first + s.nt - 1);
        int nparts = 0;
        for (int c = c1; c <= c2; ++c) nparts += P.empty(c) ? 0 : 1;
        __threadfence();
        __syncwarp();
        int merge = 0;
        if (lane == 0) merge = atomicAdd(p.tickets + s.bh, 1) == nparts - 1;
        merge = __shfl_sync(0xffffffffu, merge, 0);
        if (merge) {
          __threadfence();
          // all heads at once: the parts' maxima (lane l takes the parts l, l + 32, ...),
          // then channels 4 lane .. 4 lane + 3 of every head, the parts' loads issued
          // kBatch at a time so that their latencies overlap
          constexpr int kBatch = G <= 2 ? 4 : (G == 4 ? 2 : 1);
          float M[G];
#pragma unroll
          for (int j = 0; j < G; ++j) M[j] = -INFINITY;
          for (int k = lane, c = c1; c <= c2; ++c) {
            if (P.empty(c)) continue;
            if (k == 0) {
              const int sl = P.start(c) >= s.first ? 2 * c : 2 * c + 1;
#pragma unroll
              for (int j = 0; j < G; ++j)
                M[j] = fmaxf(M[j], __ldcg(p.part_ml + 2 * (static_cast<int64_t>(sl) * G + j)));
              k = 32;
            }
            --k;
          }
#pragma unroll
          for (int j = 0; j < G; ++j)
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) M[j] = fmaxf(M[j], __shfl_xor_sync(0xffffffffu, M[j], off));
          float Lsum[G];
          float4 ov[G];
#pragma unroll
          for (int j = 0; j < G; ++j) {
            Lsum[j] = 0.0f;
            ov[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          }
          bool nan = false;
          int c = c1;
          while (c <= c2) {
            float4 os[kBatch][G];
            float2 ml[kBatch][G];
            int nb = 0;
            for (; c <= c2 && nb < kBatch; ++c) {
              if (P.empty(c)) continue;
              const int sl = P.start(c) >= s.first ? 2 * c : 2 * c + 1;
#pragma unroll
              for (int k = 0; k < kBatch; ++k)
                if (k == nb) {
#pragma unroll
                  for (int j = 0; j < G; ++j) {
                    const int64_t prow = static_cast<int64_t>(sl) * G + j;
                    os[k][j] = __ldcg(reinterpret_cast<const float4*>(p.part_o + prow * kHeadDim) + lane);
                    ml[k][j] = __ldcg(reinterpret_cast<const float2*>(p.part_ml) + prow);
                  }
                }
              ++nb;
            }
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
              if (k >= nb) break;
#pragma unroll
              for (int j = 0; j < G; ++j) {
                const float4 o4 = os[k][j];
                nan |= o4.x != o4.x || o4.y != o4.y || o4.z != o4.z || o4.w != o4.w;
                const float f = M[j] == -INFINITY || ml[k][j].x == -INFINITY ? 0.0f : exp2f(ml[k][j].x - M[j]);
                Lsum[j] = fmaf(ml[k][j].y, f, Lsum[j]);
                ov[j].x = fmaf(o4.x, f, ov[j].x);
                ov[j].y = fmaf(o4.y, f, ov[j].y);
                ov[j].z = fmaf(o4.z, f, ov[j].z);
                ov[j].w = fmaf(o4.w, f, ov[j].w);
              }
            }
          }
#pragma unroll
          for (int j = 0; j < G; ++j) {
            const int64_t orow = static_cast<int64_t>(s.b) * p.Hq + hq0 + j;
            const float inv = p.ML ? 1.0f : (Lsum[j] > 0.0f ? 1.0f / Lsum[j] : 0.0f);
            const float nanv = __int_as_float(0x7fc00000);
            const float4 o = nan ? make_float4(nanv, nanv, nanv, nanv)
                                 : make_float4(ov[j].x * inv, ov[j].y * inv, ov[j].z * inv, ov[j].w * inv);
            reinterpret_cast<float4*>(p.O + orow * kHeadDim)[lane] = o;
            if (p.ML && lane == 0) {
              p.ML[2 * orow] = M[j];
              p.ML[2 * orow + 1] = Lsum[j];
            }
          }
          if (lane == 0) p.tickets[s.bh] = 0;  // leave the counter at zero for the next call
        }
      }
    }
  } else {
    // ============================================================== consumers
    const int r = lane >> 2, q = lane & 3;     // MMA fragment coordinates
    const int tp = lane & 7, gq = lane >> 3;   // value B-operand builder: token pair, value group
    const uint32_t mask_a0 = 0x01010101u << (2 * q), mask_a2 = mask_a0 << 1;
    // score MMA columns 2q, 2q+1 hold limbs 0,1 (q even) or 2,3 (q odd) of head 2t + q/2
    const float limb_w = (q & 1) ? 65536.0f : 1.0f;
    float* Sw = reinterpret_cast<float*>(smem + L.sbuf) + warp * G * kSStride;        // [G][kSStride]
    uint32_t* Ww = reinterpret_cast<uint32_t*>(smem + L.wbuf) + warp * 2 * G * kWStride;  // [2G][kWStride]
    // ldmatrix row addresses of the value codes, relative to the 16-token step:
    // lane l gives row (token 8 (l >> 3 & 1) + (l & 7), group 2 call + (l >> 4)); the
    // chunk swizzle reads token bits 1-2 only, so the step's 16 u tokens leave it unchanged
    uint32_t voff[2];
#pragma unroll
    for (int call = 0; call < 2; ++call) {
      const int tok = 8 * ((lane >> 3) & 1) + (lane & 7), grp = 2 * call + (lane >> 4);
      voff[call] = static_cast<uint32_t>(tok * (kHeadDim / 2) + 16 * vcode_chunk(tok, grp));
    }
    const float c_in0 = kSqrtHalfPi / static_cast<float>(m);
    const float c_out0 = m_out > 0 ? kSqrtHalfPi / static_cast<float>(m_out) : 0.0f;

    uint32_t fri[NTS][FRI][2], fro[NTS][FRO][2];
    // per N-tile t (head 2t + q/2): weights of this lane's limb sums and halves of the bias
    float cin2[NTS], cout2[NTS], bxi[NTS], bxo[NTS];
    int gs_base = 0;  // ring stages of the segments before the current one
    int gt_base = 0;  // tiles of the segments before the current one (tiles go round-robin to the warps)
    bool ok = true;
    SegIter it = seg0;
    Seg sg;

    while (it.next(p, sg)) {
      const int il = sg.il;
      const int qb = il % kNQ, cb = il % NB;
      const int n_tile = sg.n_tile();
      const int seg_t0 = sg.t0(), seg_t1 = sg.t1();
      // ---- query block of this segment
      if (ok && !mbar_wait(&qfull[qb], (il / kNQ) & 1, lim)) ok = false;
      const int first = (warp - gt_base % NC + NC) % NC;  // this warp's first tile of the segment
      const bool works = ok && first < n_tile;
      // fragment pair (t, kk) of this lane: one 8-byte load (b0, b1)
      const uint2* qfr = reinterpret_cast<const uint2*>(smem + L.qbuf + qb * L.qblock) + lane * NTS;
      const uint4* qfr4 = reinterpret_cast<const uint4*>(smem + L.qbuf + qb * L.qblock) + lane;  // NTS == 2
      if (works) {
        if (FR) {
#pragma unroll
          for (int t = 0; t < NTS; ++t) {
#pragma unroll
            for (int kk = 0; kk < FRI; ++kk)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint2 f = kk < wpt ? qfr[kk * 32 * NTS + t] : make_uint2(0u, 0u);
                fri[t][kk][h] = h ? f.y : f.x;
              }
#pragma unroll
            for (int kk = 0; kk < FRO; ++kk)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint2 f = kk < wpo ? qfr[(wpt + kk) * 32 * NTS + t] : make_uint2(0u, 0u);
                fro[t][kk][h] = h ? f.y : f.x;
              }
          }
        }
        const unsigned char* tail = smem + L.qbuf + qb * L.qblock + 4 * NTS * KK * 64;
        const int* Fs = reinterpret_cast<const int*>(tail);
        const long long* sums = reinterpret_cast<const long long*>(tail + 8 * G);
#pragma unroll
        for (int t = 0; t < NTS; ++t) {
          const int hd = min(2 * t + (q >> 1), G - 1);
          const float cin = ldexpf(c_in0, -Fs[2 * hd]), cout = ldexpf(c_out0, -Fs[2 * hd + 1]);
          cin2[t] = 2.0f * limb_w * cin;
          cout2[t] = 2.0f * limb_w * cout;
          bxi[t] = 0.5f * cin * __ll2float_rn(sums[2 * hd]);
          bxo[t] = 0.5f * cout * __ll2float_rn(sums[2 * hd + 1]);
        }
      }
      if (FR) {  // fragments are in registers: release the query block now
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfree[qb]);
      }

      // ---- running state of this warp for this segment
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
        for (int P2 = 0; P2 < 2; ++P2)
#pragma unroll
          for (int v = 0; v < NTV; ++v)
#pragma unroll
            for (int k = 0; k < 4; ++k) vacc[g][P2][v][k] = 0.0f;

      for (int s = first; works && ok && s < n_tile; s += NC) {
        const int gs = gs_base + s / kStageTiles;
        const int fill = by_nstage.div(gs), slot = by_nstage.mod(gs, fill);
        if (!seq_wait(&fill_seq[slot], fill, lim) || !mbar_wait(&full[slot], fill & 1, lim)) {
          ok = false;
          break;
        }
        const unsigned char* stg = smem + L.stages + (slot * kStageTiles + s % kStageTiles) * ST.bytes;
        const int tile0 = seg_t0 + s * kTT;             // first token of the tile
        const int n_valid = min(kTT, seg_t1 - tile0);   // >= 1
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
            if constexpr (!FR && NTS == 2) {  // both N-tiles' fragments in one load
              const uint4 f = qfr4[kk * 32];
              mma_u8s8(ai[j][0], a0, a1, a2, a3, f.x, f.y);
              mma_u8s8(ai[j][1], a0, a1, a2, a3, f.z, f.w);
            } else {
#pragma unroll
              for (int t = 0; t < NTS; ++t) {
                const uint2 f = FR ? make_uint2(fri[t][FR ? kk : 0][0], fri[t][FR ? kk : 0][1]) : qfr[kk * 32 * NTS + t];
                mma_u8s8(ai[j][t], a0, a1, a2, a3, f.x, f.y);
              }
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
                  if constexpr (!FR && NTS == 2) {
                    const uint4 f = qfr4[(wpt + ko) * 32];
                    mma_u8s8(ao[j][0], a0, a1, a2, a3, f.x, f.y);
                    mma_u8s8(ao[j][1], a0, a1, a2, a3, f.z, f.w);
                  } else {
#pragma unroll
                    for (int t = 0; t < NTS; ++t) {
                      const uint2 f =
                          FR ? make_uint2(fro[t][FR ? ko : 0][0], fro[t][FR ? ko : 0][1]) : qfr[(wpt + ko) * 32 * NTS + t];
                      mma_u8s8(ao[j][t], a0, a1, a2, a3, f.x, f.y);
                    }
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
              // <sq, sign> = 2 * sum_{bit set} - sum_all, in sq units by 2^-F (in cin2, cout2, bxi, bxo).
              // Each limb pair is exact in int32; the two pairs of a head sit in lanes q, q ^ 1, so
              // each lane weighs its pair (and half the bias) and one shuffle adds the halves.
              const float pi_r = static_cast<float>(ai[j][t][0] + 256 * ai[j][t][1]);
              const float pi_r8 = static_cast<float>(ai[j][t][2] + 256 * ai[j][t][3]);
              const float po_r = static_cast<float>(ao[j][t][0] + 256 * ao[j][t][1]);
              const float po_r8 = static_cast<float>(ao[j][t][2] + 256 * ao[j][t][3]);
              float s_r = fmaf(n_r.x, fmaf(cin2[t], pi_r, -bxi[t]), n_r.y * fmaf(cout2[t], po_r, -bxo[t]));
              float s_r8 = fmaf(n_r8.x, fmaf(cin2[t], pi_r8, -bxi[t]), n_r8.y * fmaf(cout2[t], po_r8, -bxo[t]));
              // lanes q, q ^ 1 swap halves: the even lane totals row r, the odd one row r + 8
              const bool odd = (q & 1) != 0;
              const float tot = (odd ? s_r8 : s_r) + __shfl_xor_sync(0xffffffffu, odd ? s_r : s_r8, 1);
              const int hd = 2 * t + (q >> 1);
              if (hd < G) Sw[hd * kSStride + 16 * u + r + (odd ? 8 : 0)] = tot;
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
            float* gsc = p.scores + (static_cast<int64_t>(sg.b) * p.Hq + sg.hk * G + h) * p.score_stride + tile0;
            if (v0) gsc[lane] = s0;
            if (v1) gsc[lane + 32] = s1;
          }
          // slots past the length may hold anything: they leave as -inf, p = 0
          const float l0 = v0 ? s0 * p.sm_scale_log2 : -INFINITY;
          const float l1 = v1 ? s1 * p.sm_scale_log2 : -INFINITY;
          float mx;  // the warp's maximum in one instruction (exact, like the fmaxf butterfly)
          asm("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(mx) : "f"(fmaxf(l0, l1)));
          const float new_m = fmaxf(run_m[h], mx);  // finite: token 0 of the tile is valid
          alpha[h] = ex2_ftz(run_m[h] - new_m);
          rescale |= alpha[h] != 1.0f;
          const float p0 = ex2_ftz(l0 - new_m), p1 = ex2_ftz(l1 - new_m);
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
              for (int P2 = 0; P2 < 2; ++P2)
#pragma unroll
                for (int k = 0; k < 4; ++k) vacc[g][P2][v][k] *= a;
          }
        }
        __syncwarp();
        // ---------------- values: 4 steps of 16 tokens
        const uint32_t code_base = smem_u32(stg + ST.vcode);
        const uint32_t* szw = reinterpret_cast<const uint32_t*>(stg + ST.vsz);  // [64][4] (scale, zero) fp16 pairs
#pragma unroll 1
        for (int u = 0; u < 4; ++u) {
          // codes first: they do not depend on the B operand built below
          // matrices: (group 2c, tokens 0-7), (2c, 8-15), (2c+1, 0-7), (2c+1, 8-15) of the 16
          uint32_t R[2][4];
          if constexpr (VB == 2) {
            // 2-bit codes: thread (r, q) reads the bytes of tokens 2q, 2q+1 of each
            // matrix from line (group, r) and spreads each 2-bit code into the
            // nibble the 4-bit path expects (codes 0..3 in the same fp16 scheme)
#pragma unroll
            for (int call = 0; call < 2; ++call)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int tok = 16 * u + 8 * (k & 1) + 2 * q;
                const int grp = 2 * call + (k >> 1);
                const uint32_t b2 = *reinterpret_cast<const unsigned short*>(stg + ST.vcode + v2_line(grp, r) + tok);
                const uint32_t x = __byte_perm(b2, 0u, 0x4140);  // byte 0 -> bits 0-7, byte 1 -> bits 16-23
                const uint32_t t4 = (x | (x << 4)) & 0x0F0F0F0Fu;
                R[call][k] = (t4 | (t4 << 2)) & 0x33333333u;
              }
          } else {
#pragma unroll
            for (int call = 0; call < 2; ++call)
              ldmatrix_x4_trans(R[call], code_base + 16 * u * (kHeadDim / 2) + voff[call]);
          }
          {  // B operand: w = p * scale as fp16 hi + lo for tokens 16u + 2tp, +1 and group gq
            const int t0i = 16 * u + 2 * tp;
            const uint32_t sz0 = szw[t0i * 4 + gq], sz1 = szw[(t0i + 1) * 4 + gq];
            const bool ok0 = t0i < n_valid, ok1 = t0i + 1 < n_valid;
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&sz0));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&sz1));
            const float sc0 = ok0 ? f0.x : 0.0f, z0 = ok0 ? f0.y : 0.0f;
            const float sc1 = ok1 ? f1.x : 0.0f, z1 = ok1 ? f1.y : 0.0f;
            const unsigned long long sc01 = f32x2_pack(sc0, sc1);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float2 pp = *reinterpret_cast<const float2*>(Sw + h * kSStride + t0i);
              // w = p * scale and its fp16 residual, two tokens per pair instruction
              unsigned long long w01, r01;
              asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(w01) : "l"(f32x2_pack(pp.x, pp.y)), "l"(sc01));
              const __half2 hi = __floats2half2_rn(f32x2_lo(w01), f32x2_hi(w01));
              const float2 hf = __half22float2(hi);
              asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r01) : "l"(w01), "l"(f32x2_pack(hf.x, hf.y)));
              const __half2 lo = __floats2half2_rn(f32x2_lo(r01), f32x2_hi(r01));
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
      gs_base += sg.n_stage();
      gt_base += n_tile;
      if (!ok) {
        atomicExch(flag, 1);
        atomicOr(p.hdr + 2, kDecodeErrTimeout);
      }
      if (!FR) {  // fragments were read from the query block until now
        __syncwarp();
        if (lane == 0) mbar_arrive(&qfree[qb]);
      }

      // ---- this warp's partial for the segment into combine buffer cb
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) zacc[h] += __shfl_xor_sync(0xffffffffu, zacc[h], off);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) run_l[h] += __shfl_xor_sync(0xffffffffu, run_l[h], off);
      }
      if (ok && il >= NB && !mbar_wait(&cfree[cb], ((il / NB) - 1) & 1, lim)) {
        ok = false;
        atomicExch(flag, 1);
        atomicOr(p.hdr + 2, kDecodeErrTimeout);
      }
      float* cw = reinterpret_cast<float*>(smem + L.comb) + (cb * NC + warp) * G * kPartStride;  // [G][kPartStride]
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int P2 = 0; P2 < 2; ++P2)
#pragma unroll
          for (int v = 0; v < NTV; ++v) {
            const int hd = 4 * v + q;
            if (hd < G) {
              const int d = 32 * g + 4 * r + 2 * P2;
              // rows 0-7 of the value MMA took low nibbles (n 2^-24), rows 8-15 high ones (n 2^-20)
              cw[hd * kPartStride + d] = (vacc[g][P2][v][0] + vacc[g][P2][v][1]) * kNibLoScale;
              cw[hd * kPartStride + d + 1] = (vacc[g][P2][v][2] + vacc[g][P2][v][3]) * kNibHiScale;
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

}

template <int G, int WPT_MAX, int WPO_MAX, bool EXACT, int VB>
cudaError_t launch_cfg(const DecodeParams& p0, cudaStream_t s) {
  constexpr int WPO_A = WPO_MAX > 0 ? WPO_MAX : 1;
  constexpr bool FR = Shape<G>::NTS * (WPT_MAX + WPO_A) * 2 <= Shape<G>::FRAG_BUDGET;
  DecodeParams p = p0;
  p.nstage = decode_nstage<G>(p.m, p.m_out, p.tl.vbits);
  if (p.nstage < 2) return cudaErrorInvalidConfiguration;
  const Smem L(G, Shape<G>::NC, Shape<G>::NB, p.m, p.m_out, p.nstage, p.tl.vbits);
  if (!L.aligned()) return cudaErrorInvalidConfiguration;
  const size_t smem = static_cast<size_t>(L.total);
  auto kern = decode_kernel<G, WPT_MAX, WPO_MAX, FR, EXACT, VB>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  // the prep kernel: one CTA per (sequence, kv head)
  constexpr int WMAX_PREP = (WPT_MAX + WPO_A + kPrepWarps - 1) / kPrepWarps;
  decode_prep_kernel<G, WMAX_PREP><<<static_cast<unsigned>(p.B * p.Hkv), kPrepWarps * 32, 0, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM at most (the shared memory holds one); it may
  // start before the prep grid ends and waits for it where it needs its results
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.grid));
  cfg.blockDim = dim3(Shape<G>::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

// Exact word counts for m in {128, 256, 512} with m_out = 64, else bounds;
// 2-bit value codes: exact counts for m = 256, m_out = 64, else bounds.
template <int G>
cudaError_t launch_g(const DecodeParams& p, cudaStream_t s) {
  const int wpt = p.m / 32, wpo = p.m_out / 32;
  if (p.tl.vbits == 2) {
    if (wpo == 2 && wpt == 8) return launch_cfg<G, 8, 2, true, 2>(p, s);
    if (wpo == 0) return launch_cfg<G, 16, 0, false, 2>(p, s);
    return launch_cfg<G, 16, 8, false, 2>(p, s);
  }
  if (wpo == 2) {
    if (wpt == 4) return launch_cfg<G, 4, 2, true, 4>(p, s);
    if (wpt == 8) return launch_cfg<G, 8, 2, true, 4>(p, s);
    if (wpt == 16) return launch_cfg<G, 16, 2, true, 4>(p, s);
  }
  if (wpo == 0) return launch_cfg<G, 16, 0, false, 4>(p, s);
  return launch_cfg<G, 16, 8, false, 4>(p, s);
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
