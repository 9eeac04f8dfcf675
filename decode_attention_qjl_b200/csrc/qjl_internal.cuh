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

// sqrt(pi/2) in fp32
constexpr float kSqrtHalfPi = 1.2533141373155003f;
constexpr float kLog2e = 1.4426950408889634f;

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
  uint32_t* kbits;             // [B, Hkv, cap, m/32]
  uint32_t* kbits_out;         // [B, Hkv, cap, m_out/32]
  __half* knorm;               // [B, Hkv, cap, 2]
  double* energy;              // workspace [B, Hkv, d] (prefill)
  float guard;
};

struct ValuesParams {
  const void* V;
  int64_t sb, sh, st;
  int B, Hkv, T, cap;
  const int32_t* t_start;
  uint8_t* vcode;  // [B, Hkv, cap, d/2]
  __half* vsz;     // [B, Hkv, cap, d/32, 2]
};

struct DecodeParams {
  const void* Q;  // [B, Hq, d]
  int B, Hq, Hkv, T, cap;
  const int32_t* seqlens;
  int m, m_out, n_out;
  const __nv_bfloat16* S;
  const __nv_bfloat16* S_out;
  const int32_t* idx;
  const uint32_t* kbits;
  const uint32_t* kbits_out;
  const __half* knorm;
  const uint8_t* vcode;
  const __half* vsz;
  float sm_scale_log2;  // sm_scale * log2(e)
  float* O;             // [B, Hq, d]
  float* scores;        // [B, Hq, T] or null
  int splits;           // token splits per (b, kv head)
  int chunk;            // tokens per split
  float* part_o;        // [B, Hq, splits, d]
  float* part_ml;       // [B, Hq, splits, 2]
  int* tickets;         // [B, Hkv]
};

// Launchers (return the cudaGetLastError() of the launches).
cudaError_t launch_quantize_values(const ValuesParams& p, qjl_dtype dt, cudaStream_t s);
cudaError_t launch_channel_energy(const KeysParams& p, qjl_dtype dt, cudaStream_t s);
cudaError_t launch_select_outliers(const KeysParams& p, cudaStream_t s);
cudaError_t launch_sketch_keys(const KeysParams& p, qjl_dtype dt, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams& p, qjl_dtype dt, cudaStream_t s);

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
