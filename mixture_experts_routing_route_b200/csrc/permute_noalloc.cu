// moe_permute_noalloc: moe_permute for callers that cannot allocate device
// memory, for example code that runs where the CUDA allocator is not
// reachable or not allowed (a host library handed only pre-allocated tensors,
// a runtime whose memory pool is fixed before the first call, a plugin in a
// process that forbids cudaMalloc after start-up). It needs no workspace: the
// permute's scratch (the control block with the device error word, and the
// per-slot rank buffer) lives in a file-scope static device array of a fixed
// size, which every GPU that loads this library holds until the process exits.
//
// The array is shared by every call on a device and keeps the last call's
// contents. Calls that overlap on the GPU (two streams, or two host threads)
// race on it and give wrong results; serialise them. The control block (error
// word and barrier words) is cleared at the start of each call; the rank
// buffer needs no clearing (every slot's rank is written before it is read).
// The first call on a device may load this library's device code (the CUDA
// runtime loads modules lazily), and loading allocates device memory, this
// array included: a caller that must not allocate makes one call at start-up.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kNoallocMaxSlots = MOE_PERMUTE_NOALLOC_MAX_SLOTS;
constexpr size_t kNoallocCtlWords = sizeof(Control) / 4;

// [control block (256 B)] [rank of each slot (kNoallocMaxSlots int32)]
static __device__ __align__(256) int32_t g_permute_scratch[kNoallocCtlWords + kNoallocMaxSlots];

// Device address of the static scratch on the current device. In host code
// g_permute_scratch is only a host-side stand-in for the symbol, never a
// device address, so the address must come from cudaGetSymbolAddress, called
// with the caller's device current. It is looked up on every call (a host-side
// table lookup once the module is loaded) rather than cached: after a
// cudaDeviceReset the module is loaded again and the array may move.
cudaError_t scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
  if (e != cudaSuccess) return e;
  if (p == nullptr) return cudaErrorInvalidSymbol;
  *out = p;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_permute_noalloc(const int32_t* topk_idx, int T, int k, int E,
                                            int64_t capacity, int32_t* counts, int32_t* bins,
                                            int32_t* sorted_slot, int32_t* slot_to_row,
                                            int32_t* row_slot, uint8_t* drop_mask,
                                            int32_t* kept_counts, int32_t* seg_offsets,
                                            uint32_t* device_error, moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MOE_ERR_INVALID;
  const long long S = static_cast<long long>(T) * k;
  if (S > kNoallocMaxSlots) return MOE_ERR_WORKSPACE;  // beyond the static scratch
  const void* need[] = {counts, bins, kept_counts, seg_offsets};
  for (const void* p : need) {
    if (p == nullptr) return MOE_ERR_NULL;
    if (!aligned16(p)) return MOE_ERR_ALIGN;
  }
  if (S > 0) {
    const void* need_s[] = {topk_idx, sorted_slot, slot_to_row, drop_mask};
    for (const void* p : need_s) {
      if (p == nullptr) return MOE_ERR_NULL;
      if (!aligned16(p)) return MOE_ERR_ALIGN;
    }
    if (moe_rows_max(T, k, E, capacity) > 0) {
      if (row_slot == nullptr) return MOE_ERR_NULL;
      if (!aligned16(row_slot)) return MOE_ERR_ALIGN;
    }
  }
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Control* ctl = static_cast<Control*>(scratch);
  int32_t* rank = static_cast<int32_t*>(scratch) + kNoallocCtlWords;
  if (cudaMemsetAsync(ctl, 0, sizeof(Control), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_permute_single(topk_idx, T, k, E, capacity, counts, bins, sorted_slot, slot_to_row,
                            row_slot, drop_mask, kept_counts, seg_offsets, rank, ctl,
                            s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (device_error != nullptr &&
      cudaMemcpyAsync(device_error, &ctl->err, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
