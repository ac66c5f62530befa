// decode_noalloc.cu -- routed_attention_decode for callers that cannot allocate
// device memory.
//
// The split-K decode needs a small scratch area for per-split partial results
// (running max, running sum and partial output of every query head).  The
// regular entry point takes that scratch from the caller as a workspace.  This
// variant keeps it in a fixed file-scope device array instead, so the caller
// passes only inputs and outputs.  The array is TRA_NOALLOC_SCRATCH_BYTES on
// every GPU that loads the library and stays reserved until the process exits.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/tra.h"
#include "tra_launch.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[TRA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];  // device address of g_decode_scratch, per device

// In host code `g_decode_scratch` names a host-side stand-in, not GPU memory, so
// the device address is looked up once per device (with that device current).
tra_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tra::report_error(TRA_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return tra::report_error(TRA_ERR_UNSUPPORTED, "device ordinal out of range for the fixed scratch table");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr)
      return tra::report_error(TRA_ERR_CUDA, "cudaGetSymbolAddress of the decode scratch failed");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TRA_OK;
}

}  // namespace

extern "C" tra_status routed_attention_decode_noalloc(
    const tra_shape* prefill_shape, const tra_policy* policy, const uint16_t* q,
    const uint16_t* k_new, const uint16_t* v_new, const tra_qtiles* cache, const int32_t* row_ptr,
    const uint32_t* entries, uint16_t* k_tail, uint16_t* v_tail, int32_t* tail_len_dev,
    int32_t tail_cap, float softmax_scale, uint16_t* out, int32_t* status_dev, void* stream) {
  if (!prefill_shape) return tra::report_error(TRA_ERR_INVALID, "shape is NULL");
  // The arrival counters sit in a fixed area at the start of the array for every shape
  // with B * (Hkv + 1) <= TRA_NOALLOC_MAX_COUNTERS; a larger shape would put them where
  // earlier calls left partial results, which need not be zero.
  if ((long long)prefill_shape->B * ((long long)prefill_shape->Hkv + 1) > TRA_NOALLOC_MAX_COUNTERS) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "B * (Hkv + 1) = %lld exceeds %d, the arrival counters the fixed scratch keeps at "
             "zero; use routed_attention_decode with a caller workspace",
             (long long)prefill_shape->B * ((long long)prefill_shape->Hkv + 1),
             (int)TRA_NOALLOC_MAX_COUNTERS);
    return tra::report_error(TRA_ERR_UNSUPPORTED, msg);
  }
  const size_t need = tra_decode_workspace_bytes(prefill_shape->B, prefill_shape->Hq,
                                                 prefill_shape->Hkv, prefill_shape->d);
  if (need > TRA_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "decode needs %zu bytes of scratch but the no-allocation entry point has a fixed "
             "%zu bytes; use routed_attention_decode with a caller workspace",
             need, (size_t)TRA_NOALLOC_SCRATCH_BYTES);
    return tra::report_error(TRA_ERR_UNSUPPORTED, msg);
  }
  void* scratch = nullptr;
  tra_status st = scratch_address(&scratch);
  if (st != TRA_OK) return st;
  // The scratch starts zero-filled (static storage) and every call leaves its
  // arrival counters at zero again (they stay in the fixed counter area checked
  // above); the partials behind them are written before they are read.  The regular entry point validates all other arguments and
  // enqueues the same kernel.
  return routed_attention_decode(prefill_shape, policy, q, k_new, v_new, cache, row_ptr, entries,
                                 k_tail, v_tail, tail_len_dev, tail_cap, softmax_scale, out,
                                 scratch, TRA_NOALLOC_SCRATCH_BYTES, status_dev, stream);
}
