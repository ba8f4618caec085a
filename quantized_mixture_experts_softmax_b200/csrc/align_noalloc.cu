// moe_align_noalloc: the token-to-expert alignment of moe_align for callers that cannot
// allocate device memory and have no workspace to hand over.  Examples: a plugin running
// inside a host framework that owns every device buffer, or a deployment whose device memory
// budget is fixed at start-up.  cudaMalloc may also synchronise the whole device, which some
// latency-sensitive callers cannot afford.
//
// The alignment kernels need one scratch array: a histogram of experts for every 512-pair chunk
// of the input, ceil(T*k/512) * E int32 values.  Here that scratch is a fixed array in the
// library's own device memory (kNoAllocScratchInts int32 = 512 KiB), which every GPU that
// loads the library keeps until the process exits.  Calls that need more are rejected with
// MOE_ERR_UNSUPPORTED.
//
// Host code cannot pass the array's name to a kernel: on the host that name is only a
// stand-in, not a device address.  Each call looks up the array's device address on the
// current device with cudaGetSymbolAddress (a lookup, no allocation) and remembers it per
// device; a call made while its stream is being captured into a CUDA graph uses the remembered
// address instead, so make the first call on each device before any stream capture.  Looking
// the address up again on every uncaptured call keeps it right after cudaDeviceReset, which
// reloads the library's device code, possibly at another address.  All calls share the one
// array.  Each call overwrites every scratch entry it
// reads, so leftovers from an earlier call never matter, but calls that overlap on the GPU
// (different streams, or several host threads) race on the array and must be serialised by
// the caller.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr size_t kNoAllocScratchInts = 131072;  // 512 KiB
static __device__ __align__(256) int32_t g_align_scratch[kNoAllocScratchInts];

std::mutex g_scratch_mu;

int32_t* g_scratch_addr[64];  // per device: the address the last uncaptured call looked up

moe_status_t scratch_for_current_device(cudaStream_t stream, int32_t** out) {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return MOE_ERR_CUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (cs == cudaStreamCaptureStatusNone || g_scratch_addr[d] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_align_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[d] = static_cast<int32_t*>(p);
  }
  *out = g_scratch_addr[d];
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_align_noalloc(const int32_t* topk_ids, int T, int k, int E, int align,
                                          int32_t* expert_counts, int32_t* expert_offsets, int32_t* sorted_ids,
                                          int32_t* inv_pos, cudaStream_t stream) {
  using namespace moe;
  if (T < 1 || k < 1 || E < 1 || E > 1024 || align < 1 || (int64_t)T * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)moe_align_capacity(T, k, E, align) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if ((size_t)align_blocks(T, k) * (size_t)E > kNoAllocScratchInts) return MOE_ERR_UNSUPPORTED;
  if (!aligned(topk_ids, 4) || !aligned(expert_counts, 4) || !aligned(expert_offsets, 4) || !aligned(sorted_ids, 4) ||
      !aligned(inv_pos, 4))
    return MOE_ERR_INVALID_ARG;
  if (moe_status_t st = check_device()) return st;
  int32_t* scratch = nullptr;
  if (moe_status_t st = scratch_for_current_device(stream, &scratch)) return st;
  const cudaError_t e = launch_align(topk_ids, T, k, E, align, expert_counts, expert_offsets, sorted_ids, inv_pos,
                                     scratch, nullptr, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
