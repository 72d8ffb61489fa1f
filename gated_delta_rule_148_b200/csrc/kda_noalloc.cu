// kda_prefill_noalloc: kda_prefill without any caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc at the point where they
// run the operator -- an engine whose device memory is budgeted and owned
// up front by a host framework that hands each operator only its input and
// output tensors, or a latency-critical serving loop in which cudaMalloc and
// cudaFree are not allowed because they may synchronise the whole device and
// stall every other stream.  Such a caller has nowhere to get the prefill's
// scratch from, so this entry point takes it from a fixed array compiled into
// the library.
//
// The scratch is the per-sequence span table that the pad pre-pass writes
// (one SeqSpan per sequence) and the main kernel reads; it is only touched
// when a pad mask is given.  Every entry a call reads is written earlier by
// the same call, so nothing has to be cleared between calls.
//
// Rules for callers:
//   * the array is KDA_NOALLOC_MAX_SEQS spans (64 KiB) and is held by every
//     GPU that loads the library until the process exits; a batch with more
//     sequences is rejected with KDA_ERR_INVALID_ARG before anything runs;
//   * all calls on a device share the one array and it keeps the last call's
//     contents, so two calls whose kernels overlap on the GPU (different
//     streams without ordering between them) race on it: order them;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current); make that first call
//     before any stream capture.
// No cudaMalloc, cudaFree or allocating library routine is called here.
#include <atomic>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kMaxDevicesNoAlloc = 64;

static __device__ __align__(256) unsigned char
    g_noalloc_scratch[KDA_NOALLOC_MAX_SEQS * sizeof(SeqSpan)];

// Device address of g_noalloc_scratch, per device (the host-side symbol is only
// a stand-in and must never be handed to a kernel).  Two threads whose first
// calls on a device overlap both look the address up and store the same value.
std::atomic<void *> g_noalloc_ptr[kMaxDevicesNoAlloc];

kda_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesNoAlloc)
    return KDA_ERR_CUDA;
  void *cached = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (cached == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return KDA_ERR_CUDA;
    g_noalloc_ptr[dev].store(ptr, std::memory_order_release);
    cached = ptr;
  }
  *out = cached;
  return KDA_OK;
}

}  // namespace
}  // namespace kda

extern "C" kda_status kda_prefill_noalloc(const kda_prefill_args *args, void *stream) {
  if (!args) return KDA_ERR_INVALID_ARG;
  if (args->num_seqs > KDA_NOALLOC_MAX_SEQS) return KDA_ERR_INVALID_ARG;
  void *scratch = nullptr;
  const kda_status s = kda::noalloc_scratch(&scratch);
  if (s != KDA_OK) return s;
  kda_prefill_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = sizeof(kda::g_noalloc_scratch);
  return kda_prefill(&a, stream);
}
