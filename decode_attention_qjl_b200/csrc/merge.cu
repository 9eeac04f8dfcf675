// Merge of context-parallel decode parts: one part per rank, each over a
// contiguous shard of the cached tokens.
//
// softmax(x) = exp(x - M) / sum exp(x - M) for any M >= max x ("Your Brain
// Already Runs on 1-Bit Keys", "Why Truncation Kills"), so a shard's
// unnormalised output o_r = sum_t 2^(x_t - M_r) v_t, its maximum M_r and its
// sum L_r = sum_t 2^(x_t - M_r) (logits x in log2 units, as the decode kernel
// keeps them) combine exactly: with M = max_r M_r,
//   out = sum_r 2^(M_r - M) o_r / sum_r 2^(M_r - M) L_r.
// Rank r's parts start o_stride / ml_stride floats after rank r - 1's (one
// packed buffer per rank, or two arrays). One warp per (sequence, query head) row, lane l owning channels 4l .. 4l+3;
// an empty shard (M_r = -inf, L_r = 0) adds nothing, a row with no tokens in
// any shard is zero, and a NaN part (a timed-out decode) makes the row NaN.
#include "qjl_internal.cuh"

namespace qjl {
namespace {

constexpr int kMergeWarps = 8;

__global__ void __launch_bounds__(32 * kMergeWarps)
    merge_partials_kernel(const float* __restrict__ O_parts, int64_t o_stride, const float* __restrict__ ML_parts,
                          int64_t ml_stride, int R, int64_t rows, float* __restrict__ O) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  bool nan = false;
  for (int r = 0; r < R; ++r) {
    const float mr = ML_parts[r * ml_stride + 2 * row];
    nan |= mr != mr;
    M = fmaxf(M, mr);
  }
  float L = 0.0f;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (M != -INFINITY) {
    for (int r = 0; r < R; ++r) {
      const float2 ml = reinterpret_cast<const float2*>(ML_parts + r * ml_stride)[row];
      const float4 o = reinterpret_cast<const float4*>(O_parts + r * o_stride + row * kHeadDim)[lane];
      nan |= o.x != o.x || o.y != o.y || o.z != o.z || o.w != o.w;
      if (ml.x == -INFINITY) continue;
      const float f = exp2f(ml.x - M);
      L = fmaf(ml.y, f, L);
      acc.x = fmaf(o.x, f, acc.x);
      acc.y = fmaf(o.y, f, acc.y);
      acc.z = fmaf(o.z, f, acc.z);
      acc.w = fmaf(o.w, f, acc.w);
    }
  }
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  const float nanv = __int_as_float(0x7fc00000);
  reinterpret_cast<float4*>(O + row * kHeadDim)[lane] =
      nan ? make_float4(nanv, nanv, nanv, nanv) : make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

}  // namespace

cudaError_t launch_merge_partials(const float* O_parts, int64_t o_stride, const float* ML_parts, int64_t ml_stride,
                                  int R, int64_t rows, float* O, cudaStream_t s) {
  const int64_t blocks = (rows + kMergeWarps - 1) / kMergeWarps;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  merge_partials_kernel<<<static_cast<unsigned>(blocks), 32 * kMergeWarps, 0, s>>>(O_parts, o_stride, ML_parts, ml_stride, R, rows, O);
  return cudaGetLastError();
}

}  // namespace qjl
