// Attention entry point that allocates nothing.
//
// Some callers cannot allocate device memory at the point where they need
// attention: a real-time serving loop with a hard per-unit deadline, where a
// cudaMalloc/cudaFree can synchronise the device and stall the thread for an
// unbounded time, and host programs that hand all device memory to their own
// allocator and give this library none.  sfm_attention_noalloc serves them:
// the caller still passes Q, K, V and O, and the split-KV partial results
// live in a fixed array compiled into the library instead of a caller
// workspace.
//
// The array is a file-scope __device__ variable, so every GPU that loads this
// library holds it (SFM_NOALLOC_SCRATCH_BYTES) until the process exits.  In
// host code its name is only a host-side stand-in, never a device address:
// the first call on each device, with that device current, resolves the real
// address with cudaGetSymbolAddress and keeps it for that device's context (a
// cudaDeviceReset brings up a new context, with the module loaded again, and
// the next call resolves the address again).  All calls share the array and it
// keeps the last call's contents; nothing in it has to start at zero, because
// every partial the merge reads is written earlier in the same call.  A bounded
// wait that gives up inside the kernel is reported, like for every standalone
// call, through the per-device word sfm_check_call_error reads.
#include <mutex>

#include "attn.cuh"

namespace {

static_assert(SFM_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte alignment");

static __device__ __align__(256) unsigned char g_attn_scratch[SFM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct ScratchSlot {
  void* ctx = nullptr;   // the context the address belongs to
  void* ptr = nullptr;
};
ScratchSlot g_scratch_dev[kMaxDevices];

// Device address of g_attn_scratch on the current device (resolved once per
// device and context).
int scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return sfm::record_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return SFM_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  void* ctx = nullptr;
  if (sfm::current_context(&ctx)) return SFM_ECUDA;
  ScratchSlot& slot = g_scratch_dev[dev];
  if (!ctx || slot.ctx != ctx || !slot.ptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess || !p) return sfm::record_cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
    if (!ctx && (sfm::current_context(&ctx) || !ctx)) return SFM_ECUDA;
    slot.ctx = ctx;
    slot.ptr = p;
  }
  *out = slot.ptr;
  return SFM_OK;
}

}  // namespace

extern "C" {

int sfm_attention_noalloc(const void* q, const void* k, const void* v, void* o, int n_q,
                          int n_kv, int n_heads, int head_dim, int dtype, void* stream) {
  if (!q || !k || !v || !o || n_q < 1 || n_kv < 1 || n_heads < 1) return SFM_EINVAL;
  if (dtype != SFM_DTYPE_BF16 && dtype != SFM_DTYPE_FP32) return SFM_EINVAL;
  const size_t need = sfm_attention_workspace_bytes(n_q, n_kv, n_heads, head_dim, dtype);
  if (need > (size_t)SFM_NOALLOC_SCRATCH_BYTES) return SFM_ECAPACITY;
  void* scratch = nullptr;
  if (need > 0) {
    const int rc = scratch_on_current_device(&scratch);
    if (rc != SFM_OK) return rc;
  }
  return sfm_attention(q, k, v, o, n_q, n_kv, n_heads, head_dim, dtype, scratch, need, stream);
}

}  // extern "C"
