// A block entry point for callers that cannot allocate device memory.
//
// mmh3_block_forward needs a caller-provided workspace for the block's
// intermediates.  Some callers have no way to provide one: a plugin inside a
// host program that owns every device allocation through its own pool and
// gives plugins no allocator, a runtime that must not call cudaMalloc on its
// hot path because cudaMalloc synchronises the device, or a minimal embedder
// that links only this library and holds no device memory of its own beyond
// the tensors it passes in.  For them, mmh3_block_forward_noalloc runs the
// same kernels with the intermediates placed in one file-scope __device__
// array of fixed size, so the call itself allocates nothing.
//
// The array is reserved on every GPU where this library's device code is
// loaded and stays reserved until the process exits.  Its device address is
// looked up once per device (the first call on that device, with the device
// current), so that first call should be made before any stream capture.
// The address is kept together with the CUDA context that was current at
// the lookup; a call under another context on that device (after
// cudaDeviceReset, say, when the module is loaded again and the array may
// move) looks the address up again.
// All calls share the array: two calls whose kernels overlap on the GPU (for
// example on two streams without ordering) race on it and give wrong
// results.  Nothing in the array has to start at zero -- every region the
// block reads is written earlier in the same call.
#include <cstring>
#include <mutex>

#include "mmh3_internal.h"

namespace {

constexpr size_t kScratchBytes = MMH3_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code this name only stands for the symbol;
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

// Per device: the context of the last lookup and the address found there.
struct ScratchSlot {
  void* ctx;
  void* addr;
};
static ScratchSlot g_scratch[kMaxDevices] = {};
static std::mutex g_scratch_mu;

// The current CUDA context (the driver's cuCtxGetCurrent, reached through
// the runtime's entry-point query), or null if it cannot be asked.
void* current_context() {
  using GetCtx = int (*)(void**);
  static GetCtx fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCtx>(p);
  });
  void* ctx = nullptr;
  if (fn != nullptr && fn(&ctx) != 0) ctx = nullptr;
  return ctx;
}

// Device address of the scratch array on the current device, or null with
// the error recorded.
void* scratch_address(mmh3_status* st) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *st = mmh3::cuda_fail(e, "noalloc: cudaGetDevice");
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *st = mmh3::fail(MMH3_ERR_UNSUPPORTED, "noalloc: device ordinal %d above %d", dev, kMaxDevices - 1);
    return nullptr;
  }
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (slot.addr == nullptr || slot.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *st = mmh3::cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "noalloc: cudaGetSymbolAddress");
      return nullptr;
    }
    slot.ctx = ctx;
    slot.addr = p;
  }
  return slot.addr;
}

}  // namespace

extern "C" mmh3_status mmh3_block_forward_noalloc(const mmh3_dims* dims, const mmh3_block_weights* w,
                                                  float* x, int n, const mmh3_segment* segs, int n_seg,
                                                  const float* pos_dev, double sigma_v, double sigma_a,
                                                  int modulated, void* stream) {
  mmh3::clear_error();
  size_t need = 0;
  mmh3_status st = mmh3_workspace_size(dims, n, &need);
  if (st != MMH3_OK) return st;
  if (need > kScratchBytes) {
    // largest token count whose intermediates still fit, for the message
    int lo = 0, hi = n;
    while (lo < hi) {
      const int mid = lo + (hi - lo + 1) / 2;
      size_t b = 0;
      mmh3_workspace_size(dims, mid, &b);
      if (b <= kScratchBytes) lo = mid; else hi = mid - 1;
    }
    return mmh3::fail(MMH3_ERR_WORKSPACE,
                      "noalloc: %d tokens need %zu bytes of scratch, above the fixed %zu bytes; "
                      "at most %d tokens fit for these dims (use mmh3_block_forward with a workspace)",
                      n, need, kScratchBytes, lo);
  }
  void* scratch = scratch_address(&st);
  if (scratch == nullptr) return st;
  return mmh3::block_forward_impl(dims, w, x, n, segs, n_seg, pos_dev, sigma_v, sigma_a, modulated, nullptr,
                                  scratch, kScratchBytes, stream, /*profile=*/false);
}
