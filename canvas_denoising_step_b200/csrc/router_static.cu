// dg_router_topk_static: the router selection and grouping of dg_router_topk
// for callers that cannot allocate device memory.  It needs no context (a
// context allocates its weights and workspace); its scratch -- the expert
// membership bitmap, the last-block counter and the inverse permutation --
// lives in one file-scope __device__ array, present on every GPU that loads
// this library until the process exits.
#include <mutex>

#include "dg.h"
#include "dg_kernels.h"

namespace {

constexpr int kStaticMaxRows = 2048;
constexpr int kStaticMaxExperts = 256;
constexpr int kStaticMaxTopK = 8;
constexpr int kCounterWords = 64;   // counter (word 0) and error word (word 1), padded to 256 B
constexpr int kBitmapWords = kStaticMaxExperts * ((kStaticMaxRows + 31) / 32);
constexpr int kInvWords = kStaticMaxRows * kStaticMaxTopK;
constexpr int kScratchWords = kCounterWords + kBitmapWords + kInvWords;   // 131,328 bytes

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t* g_scratch_dev[kMaxDevices] = {};   // device address of the array, per device

}  // namespace

static __device__ __align__(256) uint32_t g_router_scratch[kScratchWords];

extern "C" int dg_router_topk_static(const float* logits, int n_rows, int n_experts, int top_k,
                                     int32_t* idx, float* w, int32_t* offsets, int32_t* perm,
                                     void* cuda_stream) {
  if (!logits || !idx || !w || !offsets || !perm) return DG_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(logits) & 15) return DG_ERR_INVALID_ARG;
  if (n_rows < 1 || n_rows > kStaticMaxRows) return DG_ERR_INVALID_ARG;
  if (n_experts < 4 || n_experts > kStaticMaxExperts || n_experts % 4) return DG_ERR_INVALID_ARG;
  if (top_k < 1 || top_k > kStaticMaxTopK || top_k > n_experts) return DG_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return DG_ERR_CUDA;
  }
  uint32_t* base;
  {
    // First call on this device: look up the array's device address (host code
    // must not pass the symbol itself, which is only a host-side stand-in).
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_dev[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_router_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return DG_ERR_CUDA;
      }
      g_scratch_dev[dev] = static_cast<uint32_t*>(p);
    }
    base = g_scratch_dev[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const int W = (n_rows + 31) / 32;
  // the counter, the error word and the bitmap words this call uses start at zero
  if (cudaMemsetAsync(base, 0, sizeof(uint32_t) * ((size_t)kCounterWords + (size_t)n_experts * W),
                      s) != cudaSuccess) {
    cudaGetLastError();
    return DG_ERR_CUDA;
  }
  dg::RouterArgs ra;
  memset(&ra, 0, sizeof(ra));
  ra.logits_in = logits;
  ra.splits = 1;
  ra.T = n_rows;
  ra.E = n_experts;
  ra.k = top_k;
  ra.n_shared = 0;
  ra.n_tile = 128;
  ra.idx = idx;
  ra.w = w;
  ra.counter = reinterpret_cast<int*>(base);
  ra.err = reinterpret_cast<int*>(base) + 1;
  ra.bitmap = base + kCounterWords;
  ra.inv = reinterpret_cast<int32_t*>(base + kCounterWords + kBitmapWords);
  ra.offsets_r = offsets;
  ra.perm = perm;
  if (dg::launch_router(ra, s) != cudaSuccess) {
    cudaGetLastError();
    return DG_ERR_CUDA;
  }
  return DG_OK;
}
