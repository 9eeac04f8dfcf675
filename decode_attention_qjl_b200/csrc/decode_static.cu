// qjl_decode_attention_static: decode attention whose scratch memory is a
// fixed array inside the library, for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc: a plugin running inside a host runtime
// that owns all of the device's memory and forbids its plugins to allocate, or
// a latency-critical caller that cannot accept the implicit device
// synchronisation of cudaMalloc/cudaFree. This entry point gives them decode
// attention without any allocation: the decode workspace (counters, prepared
// query sketches, partial results) lives in g_scratch below, a file-scope device array of
// kStaticScratchBytes that every GPU which loads the library holds until the
// process exits. The caller still passes its inputs and outputs.
//
// In host code the name g_scratch is only a host-side stand-in, not a device
// address: handing it to a kernel would fault or, where the GPU can reach host
// memory, silently use the wrong memory. Its device address is looked up once
// per device with cudaGetSymbolAddress (by the first call made on that device,
// with that device current) and passed on as a plain workspace pointer.
#include <mutex>
#include <string>

#include "qjl_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = QJL_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_dev[kMaxDevices] = {};  // device address of g_scratch, per device

// Device address of g_scratch on the current device, looked up on first use.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_dev[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" qjl_status qjl_decode_attention_static(qjl_ctx* ctx, const qjl_cache* cache, const void* Q,
                                                  qjl_dtype dtype, int Hq, int T, const int32_t* seqlens,
                                                  float sm_scale, float* O, float* scores, void* stream) {
  if (!ctx || !cache) {
    qjl::set_last_error("qjl_decode_attention_static: null context or cache");
    return QJL_ERR_ARG;
  }
  const size_t need = qjl_decode_workspace_bytes(ctx, cache->B, Hq, cache->Hkv, T);
  if (need > kStaticScratchBytes) {
    qjl::set_last_error("qjl_decode_attention_static: this call needs " + std::to_string(need) +
                        " bytes of scratch, more than the fixed " + std::to_string(kStaticScratchBytes) +
                        " bytes (QJL_STATIC_SCRATCH_BYTES); use qjl_decode_attention with a caller workspace");
    return QJL_ERR_WORKSPACE;
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev != qjl::ctx_device(ctx)) {
    qjl::set_last_error("qjl_decode_attention_static: the context's device must be the current device");
    return QJL_ERR_ARG;
  }
  void* scratch = nullptr;
  e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    qjl::set_last_error(std::string("qjl_decode_attention_static: scratch set-up: ") + cudaGetErrorString(e));
    return QJL_ERR_CUDA;
  }
  // The array keeps the previous call's contents; the header and the merge
  // counters at its start must be zero (the rest is written before it is read).
  const size_t zero = qjl::decode_ws_zero_bytes(ctx, cache->B, Hq, cache->Hkv);
  if (zero > 0) {
    e = cudaMemsetAsync(scratch, 0, zero, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
      qjl::set_last_error(std::string("qjl_decode_attention_static: clear: ") + cudaGetErrorString(e));
      return QJL_ERR_CUDA;
    }
  }
  return qjl_decode_attention(ctx, cache, Q, dtype, Hq, T, seqlens, sm_scale, O, scores, scratch,
                              kStaticScratchBytes, stream);
}
