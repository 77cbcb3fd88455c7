// mla_static_scratch.cu -- a decode entry point that allocates no device memory.
//
// mla_decode_kvcache needs a caller-provided workspace for the fp32 partial
// results of sequences that are split across workers.  Some callers cannot
// obtain one: for example an engine that reserves all device memory up front in
// its own arena and forbids any further cudaMalloc, or a latency-critical loop
// that must never call cudaMalloc/cudaFree (cudaFree synchronises the device).
// For them, mla_decode_kvcache_static_scratch keeps that workspace in a
// fixed-size array compiled into this library instead.
//
// What to know before using it:
//   - The array is kStaticScratchBytes (48 MiB) per GPU.  Every GPU that loads
//     this part of the library holds it until the process exits.
//   - Calls whose workspace would exceed it are rejected with
//     MLA_ERR_SCRATCH_LIMIT before anything is launched (null pointers and bad
//     sizes are reported as MLA_ERR_INVALID_ARG first).
//   - All calls on a device share the one array, and it keeps whatever the
//     last call left there.  The decode writes every partial it later reads, so
//     nothing has to start at zero; but two calls that run on the GPU at the
//     same time (different streams, or other threads) race on the array.
//     Serialise them.
//   - The first call on each device looks up the array's device address (a
//     runtime call that may load this module); make that first call before
//     any stream capture.
//   - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "mla_kernels.cuh"

namespace {

constexpr size_t kStaticScratchBytes = MLA_STATIC_SCRATCH_BYTES;
constexpr int kMaxScratchDevices = 64;

// In host code this name is only a host-side handle for the symbol, not a
// device address: the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of the array on the current device, looked up once per device.
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxScratchDevices) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr)
      return MLA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" {

int mla_decode_kvcache_static_scratch(const void* q, const void* kcache, int64_t num_blocks,
                                      const int32_t* block_table, int bt_stride,
                                      const int32_t* cache_seqlens, int batch, int s_q, int h_q,
                                      int d, int dv, float softmax_scale, int causal,
                                      const int32_t* tile_md, const int32_t* num_splits,
                                      int num_workers, void* out, float* lse,
                                      int32_t* device_status, void* stream) {
  // The argument checks of mla_decode_kvcache that do not depend on the
  // workspace come first, so that a call with a null pointer or a bad size
  // reports MLA_ERR_INVALID_ARG whatever workspace its shape would need.
  if (q == nullptr || kcache == nullptr || block_table == nullptr || cache_seqlens == nullptr ||
      tile_md == nullptr || num_splits == nullptr || out == nullptr || lse == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (d != MLA_HEAD_DIM_QK || dv != MLA_HEAD_DIM_V) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || s_q < 1 || h_q < 1 || bt_stride < 1 || num_workers < 1 || num_blocks < 1)
    return MLA_ERR_INVALID_ARG;
  const size_t need = mla_workspace_size(batch, s_q, h_q, dv, num_workers);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return MLA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const int rc = static_scratch_address(&scratch);
  if (rc != MLA_OK) return rc;
  return mla_decode_kvcache(q, kcache, num_blocks, block_table, bt_stride, cache_seqlens, batch,
                            s_q, h_q, d, dv, softmax_scale, causal, tile_md, num_splits,
                            num_workers, scratch, kStaticScratchBytes, out, lse, device_status,
                            stream);
}

}  // extern "C"
