// decode_noalloc.cu - attn_decode_noalloc: the split-KV paged decode of
// attn_decode, with its scratch (the per-split partial outputs and LSEs)
// taken from a fixed array that is part of this library instead of from a
// workspace the caller allocates.
//
// Who needs it: callers that may not allocate device memory at all. For
// example, a plugin inside a serving engine that plans all of its device
// memory once at start-up and hands each plugin only its input and output
// buffers. Another is a latency-critical decode loop that cannot afford
// cudaMalloc, which can synchronise the whole device and take unbounded
// time. Such a caller passes inputs and outputs only; the scratch comes
// from here.
//
// Rules of use:
//  - The scratch holds at most ATTN_DECODE_NOALLOC_MAX_BYTES (32 MiB). Every
//    GPU that loads the library keeps that much device memory until the
//    process exits. A call whose partials need more (attn_decode_workspace_bytes
//    for its batch, heads, head dim and split count) is refused with
//    ATTN_ERR_WORKSPACE before anything is launched.
//  - The first call on each device does a one-time set-up: it looks up the
//    device address of the array (cudaGetSymbolAddress), which may also load
//    the library's device code on that device. Make that first call before
//    any stream capture on the device. The address is remembered together
//    with the CUDA context it belongs to; if that context is replaced (after
//    cudaDeviceReset, say), the next call repeats the set-up in the new one,
//    and so should come before any capture as well.
//  - Every call on a device uses the same array, which keeps whatever the
//    previous call left there. Nothing in it has to start at zero: every
//    partial the combine step reads is written by the same call first. Calls
//    that can overlap on the GPU (on different streams, or from different
//    threads without ordering) race on the array and corrupt each other's
//    results; issue them in order on one stream.
//  - Nothing here allocates or frees device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/attn.h"

static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_DECODE_NOALLOC_MAX_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Per device: the device address of g_decode_scratch and the context in
// which it was looked up.
struct ScratchSlot {
  CUcontext ctx;
  void* addr;
};
ScratchSlot g_slots[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry-point lookup, so the
// library needs no link-time dependency on libcuda.
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  return fn;
}

// Host code cannot use g_decode_scratch directly: on the host that name is
// only a stand-in for the device variable. Its device address is looked up
// with the device current and cached with the current context; a different
// context (the old one was reset) triggers a fresh lookup, so a stale
// address is never handed to a kernel.
attn_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return ATTN_ERR_CUDA;
  if (ctx == nullptr) {
    // No context is current yet: the symbol lookup initialises the device's
    // primary context (it allocates nothing), after which it is current.
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_decode_scratch) != cudaSuccess) return ATTN_ERR_CUDA;
    if (get(&ctx) != CUDA_SUCCESS || ctx == nullptr) return ATTN_ERR_CUDA;
  }
  ScratchSlot& slot = g_slots[dev];
  if (slot.addr == nullptr || slot.ctx != ctx) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_decode_scratch) != cudaSuccess || addr == nullptr) return ATTN_ERR_CUDA;
    slot.ctx = ctx;
    slot.addr = addr;
  }
  *out = slot.addr;
  return ATTN_OK;
}

}  // namespace

extern "C" attn_status attn_decode_noalloc(const attn_decode_params* p, void* stream) {
  if (!p) return ATTN_ERR_INVALID_ARG;
  if (p->B == 0) return attn_decode(p, nullptr, 0, stream);
  const int splits = attn_decode_num_splits(p->B, p->Hq, p->Hkv, p->max_seqlen, p->num_splits);
  const size_t need = attn_decode_workspace_bytes(p->B, p->Hq * (p->q_len > 1 ? p->q_len : 1), p->D, splits);
  if (need > static_cast<size_t>(ATTN_DECODE_NOALLOC_MAX_BYTES)) return ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (attn_status st = scratch_address(&scratch)) return st;
  return attn_decode(p, scratch, static_cast<size_t>(ATTN_DECODE_NOALLOC_MAX_BYTES), stream);
}
