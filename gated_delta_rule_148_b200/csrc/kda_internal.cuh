// Internal declarations shared by the translation units of libkda.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Bits latched in the per-device error word.
enum : unsigned {
  ERR_BIT_CHECK = 1u,     // device-side argument check failed
  ERR_BIT_TIMEOUT = 2u,   // a bounded wait ran out
};

// Per-sequence span of positions a prefill kernel processes: [begin, end)
// in packed rows.  Rows of the sequence outside the span are edge pads.
struct SeqSpan {
  int begin;
  int end;
  int seq_begin;   // cu[b]
  int pad_inside;  // 1 if a pad sits strictly inside [begin, end)
};

struct PrefillParams {
  int num_seqs, N, H, dk, dv, chunk;
  const void *q, *k, *v;
  const float *log_alpha, *beta;
  const int32_t *cu;
  const uint8_t *mask;
  const float *init_state;
  void *o;
  float *final_state;
  const SeqSpan *spans;   // NULL: spans are [cu[b], cu[b+1])
  unsigned *err;          // device error word
  int gate_head;          // 1: log_alpha is [N, H] (one gate per token and head)
  long long wait_cycles;  // limit of every bounded device wait
  int fault;              // test faults (FAULT_*), 0 in normal use
  unsigned *site;         // device word: code of the first bounded wait that ran out
};

// Faults a test can plant with kda_debug_set_fault() to exercise the bounded
// waits; none of them touches memory out of bounds.
enum : int {
  FAULT_STARVE_STATE_LOADS = 1,   // the state pass issues no item loads: its waits run out
};
constexpr long long kDefaultWaitCycles = 4000000000LL;   // ~2 s at 1.9 GHz

struct DecodeParams {
  int B, H, dk, dv;
  const void *q, *k, *v;
  const float *log_alpha, *beta;
  const uint8_t *mask;
  float *state;
  void *o;
  unsigned *err;
  int gate_head;          // 1: log_alpha is [B, H]
};

struct ConvParams {
  int num_seqs, N, D, W;
  const void *x;
  const float *weight, *bias;
  const int32_t *cu;
  const uint8_t *mask;
  const float *state_in;
  float *state_out;
  void *y;
  unsigned *err;
};

struct BackwardParams {
  int num_seqs, N, H, dk, dv;
  const void *q, *k, *v;
  const float *log_alpha, *beta;
  const int32_t *cu;
  const uint8_t *mask;
  const float *init_state;
  const float *d_o, *d_final_state;
  float *gq, *gk, *gv, *gla, *gbeta, *g_init_state;
  void *ws;               // chunk index, per-chunk quantities, states at chunk starts and ends
  unsigned *err;
  int gate_head;
};

// Launchers (return a CUDA error code; argument checks happen before).
cudaError_t launch_prefill_prepass(const PrefillParams &p, bool bf16, SeqSpan *spans,
                                   cudaStream_t s);
cudaError_t launch_prefill_simt(const PrefillParams &p, bool bf16, cudaStream_t s);
cudaError_t launch_prefill_tc(const PrefillParams &p, cudaStream_t s);  // may return
                                                                          // cudaErrorNotSupported
bool prefill_tc_supported(const PrefillParams &p, bool bf16);
bool prefill_split_supported(const PrefillParams &p, bool bf16);
size_t prefill_split_workspace(int N, int B, int H);
cudaError_t launch_prefill_split(const PrefillParams &p, SeqSpan *spans, void *ws, cudaStream_t s);
// The two-kernel path's chunk index and intra kernel alone (64-row items of every chunk and head).
cudaError_t launch_split_items(const PrefillParams &p, const SeqSpan *spans, int *cbase,
                               unsigned char *items, cudaStream_t s);
// Chunks of 128 or 256 rows: 64-row items merged into chunk items, then the state pass.
bool prefill_bigchunk_supported(const PrefillParams &p, bool bf16);
size_t prefill_bigchunk_workspace(int N, int B, int H, int chunk);
cudaError_t launch_prefill_bigchunk(const PrefillParams &p, SeqSpan *spans, void *ws, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams &p, bool bf16, cudaStream_t s);
cudaError_t launch_short_conv(const ConvParams &p, bool bf16, cudaStream_t s);
size_t backward_workspace(int N, int B, int H, int dk, int dv);
cudaError_t launch_backward(const BackwardParams &p, bool bf16, cudaStream_t s);

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(((unsigned)h) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  // round to nearest even; inputs here are finite
  unsigned u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

template <bool BF16>
__device__ __forceinline__ float load_elem(const void *base, size_t idx) {
  if (BF16) return bf16_to_f32(reinterpret_cast<const uint16_t *>(base)[idx]);
  return reinterpret_cast<const float *>(base)[idx];
}

template <bool BF16>
__device__ __forceinline__ void store_elem(void *base, size_t idx, float val) {
  if (BF16) reinterpret_cast<uint16_t *>(base)[idx] = f32_to_bf16_rne(val);
  else reinterpret_cast<float *>(base)[idx] = val;
}

// Offset of log_alpha for (row, head h, channel c): [rows, H, dk] or, with a
// head-wise gate, [rows, H] (the same value for every channel).
__device__ __forceinline__ size_t la_index(size_t row, int h, int H, int dk, int c, int gate_head) {
  return gate_head ? row * H + h : (row * H + h) * dk + c;
}

// Records which bounded wait ran out first (codes listed with kda_debug_timeout_site()).
__device__ __forceinline__ void note_timeout(unsigned *site, unsigned code) {
  if (site) atomicCAS(site, 0u, code);
}

__device__ __forceinline__ bool device_error_latched(const unsigned *err) {
  return *reinterpret_cast<const volatile unsigned *>(err) != 0u;
}

}  // namespace kda
