// align_static.cu -- the routing sort without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they route a batch:
// a serving engine that reserves all free device memory for its KV cache at start-up
// and forbids later cudaMalloc calls, or code that runs while a CUDA graph is being
// captured (where cudaMalloc is not allowed) and has no workspace tensor to pass.
// chord_moe_align_noalloc serves them: the only scratch the routing sort needs (the
// per-run expert histograms of large batches) lives in the file-scope device array
// below, which exists on every device that loads this library for as long as the
// process runs. Nothing else differs from chord_moe_align.
#include <mutex>

#include "chord_internal.cuh"

namespace chord {
namespace {

// Largest scratch the routing sort may need here: per-run histograms for up to
// 2^17 flat slots (128 runs of 1024) and up to 1024 experts, plus the count and offset
// arrays: 1024*128*4 + 4096 + 4352 = 532,736 bytes.
constexpr int64_t kStaticMaxSlots = int64_t(1) << 17;
constexpr size_t kStaticScratchBytes = 576 * 1024;

static __device__ __align__(256) uint8_t g_align_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_align_scratch on the current device (looked up once per device;
// host code may not pass the symbol itself to a kernel).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_align_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace chord

using namespace chord;

extern "C" chord_status_t chord_moe_align_noalloc(const int32_t* topk_ids, int64_t T, int topk, int E,
                                                  int block_m, int32_t* sorted_ids, int32_t* expert_ids,
                                                  int32_t* num_tokens_padded, int32_t* expert_offsets,
                                                  chord_stream_t stream) {
  // the same checks, statuses and detail texts as chord_moe_align, in the same order
  clear_detail();
  chord_status_t st = check_align_args(T, topk, E, block_m);
  if (st != CHORD_OK) return st;
  if ((T > 0 && !topk_ids) || !sorted_ids || !expert_ids || !num_tokens_padded)
    return fail(CHORD_ERR_INVALID_ARG, "null routing pointer");
  // the one limit of its own: the static scratch (T*topk < 2^31 is already checked)
  if (T * topk > kStaticMaxSlots || align_workspace_bytes(T * topk, E) > kStaticScratchBytes)
    return fail(CHORD_ERR_UNSUPPORTED, "T*topk=%lld exceeds the static scratch limit of %lld slots",
                (long long)(T * topk), (long long)kStaticMaxSlots);
  if ((st = current_device(nullptr)) != CHORD_OK) return st;
  void* scratch = nullptr;
  cudaError_t err = scratch_address(&scratch);
  if (err != cudaSuccess) return cuda_fail(err, "static scratch address (cudaGetSymbolAddress)");
  const int64_t cap = T * topk + int64_t(E) * (block_m - 1);
  const int64_t nblocks = (cap + block_m - 1) / block_m;
  err = launch_align(topk_ids, T * topk, E, block_m, cap, nblocks, sorted_ids, expert_ids, num_tokens_padded,
                     expert_offsets, scratch, reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_align launch");
  return CHORD_OK;
}
