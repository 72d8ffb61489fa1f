// C ABI of libkda.so: argument validation, dispatch, device error word.
//
// Every entry point validates on the host first and launches nothing on an
// argument error.  See include/kda.h for the contract of each call.
#include <atomic>
#include <cstring>

#include "kda_internal.cuh"

namespace kda {

// Per-device error word (bits of ERR_BIT_*); kernels OR into it.
__device__ unsigned g_error_word;
// Per-device code of the first bounded wait that ran out (0: none since the last read).
__device__ unsigned g_timeout_site;

namespace {

constexpr int kMaxDevices = 64;
// Device address of g_error_word, per device.  Threads that make their first call on a
// device at the same time both look it up and store the same value.
std::atomic<unsigned *> g_err_ptr[kMaxDevices];

kda_status error_word(unsigned **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
  unsigned *cached = g_err_ptr[dev].load(std::memory_order_acquire);
  if (cached == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess || ptr == nullptr) return KDA_ERR_CUDA;
    cached = static_cast<unsigned *>(ptr);
    g_err_ptr[dev].store(cached, std::memory_order_release);
  }
  *out = cached;
  return KDA_OK;
}

std::atomic<unsigned *> g_site_ptr[kMaxDevices];

kda_status timeout_site_word(unsigned **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KDA_ERR_CUDA;
  unsigned *cached = g_site_ptr[dev].load(std::memory_order_acquire);
  if (cached == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_timeout_site) != cudaSuccess || ptr == nullptr) return KDA_ERR_CUDA;
    cached = static_cast<unsigned *>(ptr);
    g_site_ptr[dev].store(cached, std::memory_order_release);
  }
  *out = cached;
  return KDA_OK;
}

// Test faults and the bounded-wait limit (kda_debug_set_fault); process-wide.
std::atomic<int> g_fault{0};
std::atomic<long long> g_wait_cycles{kDefaultWaitCycles};

struct Range {
  const void *p;
  size_t bytes;
};

bool overlap(Range a, Range b) {
  if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
  const uintptr_t a0 = (uintptr_t)a.p, a1 = a0 + a.bytes;
  const uintptr_t b0 = (uintptr_t)b.p, b1 = b0 + b.bytes;
  return a0 < b1 && b0 < a1;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool head_dim_ok(int d) { return d == 64 || d == 128; }

size_t elem_bytes(kda_dtype t) { return t == KDA_BF16 ? 2 : 4; }

size_t spans_bytes(int num_seqs) {
  const size_t raw = sizeof(SeqSpan) * (size_t)(num_seqs > 0 ? num_seqs : 0);
  return (raw + 255) / 256 * 256;
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" {

int kda_version(void) { return (1 << 16) | 1; }

const char *kda_status_string(kda_status s) {
  switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: configuration not supported";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA runtime call failed";
    case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
    case KDA_ERR_DEVICE_CHECK: return "KDA_ERR_DEVICE_CHECK: a device-side argument check failed";
  }
  return "KDA_ERR_UNKNOWN";
}

// Whether a call may take the two-kernel tensor-core path (given enough workspace).
bool split_eligible(const kda_prefill_args *a) {
  const int chunk = a->chunk == 0 ? (a->dtype == KDA_BF16 ? 64 : 16) : a->chunk;
  return a->dtype == KDA_BF16 && a->dk == 128 && a->dv == 128 && chunk == 64 && a->num_seqs > 0 &&
         a->total_tokens >= 0 && a->H >= 1;
}

// Chunks of 128 or 256 rows: only on the tensor-core path (bf16, d_k = d_v = 128).
bool bigchunk_eligible(const kda_prefill_args *a) {
  return a->dtype == KDA_BF16 && a->dk == 128 && a->dv == 128 && (a->chunk == 128 || a->chunk == 256) &&
         a->num_seqs > 0 && a->total_tokens >= 0 && a->H >= 1;
}

size_t kda_prefill_workspace_size(const kda_prefill_args *a) {
  if (!a) return 0;
  if (bigchunk_eligible(a)) return prefill_bigchunk_workspace(a->total_tokens, a->num_seqs, a->H, a->chunk);
  if (split_eligible(a)) return prefill_split_workspace(a->total_tokens, a->num_seqs, a->H);
  return spans_bytes(a->num_seqs);
}

kda_status kda_prefill(const kda_prefill_args *a, void *stream) {
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->dtype != KDA_F32 && a->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (a->num_seqs < 0 || a->total_tokens < 0 || a->H < 1) return KDA_ERR_INVALID_ARG;
  if (a->dk <= 0 || a->dv <= 0) return KDA_ERR_INVALID_ARG;
  if (!head_dim_ok(a->dk) || !head_dim_ok(a->dv)) return KDA_ERR_UNSUPPORTED;
  int chunk = a->chunk;
  if (chunk == 0) chunk = (a->dtype == KDA_BF16) ? 64 : 16;
  const bool big = chunk == 128 || chunk == 256;
  if (chunk != 16 && chunk != 32 && chunk != 64 && !big) return KDA_ERR_UNSUPPORTED;
  if (big && (a->dtype != KDA_BF16 || a->dk != 128 || a->dv != 128)) return KDA_ERR_UNSUPPORTED;
  if (a->gate != KDA_GATE_CHANNEL && a->gate != KDA_GATE_HEAD) return KDA_ERR_INVALID_ARG;
  const bool gate_head = a->gate == KDA_GATE_HEAD;
  if (a->num_seqs == 0) return a->total_tokens == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
  if (!a->cu_seqlens) return KDA_ERR_INVALID_ARG;
  const size_t N = (size_t)a->total_tokens, H = (size_t)a->H;
  const size_t es = elem_bytes(a->dtype);
  const Range q{a->q, N * H * a->dk * es}, k{a->k, N * H * a->dk * es};
  const Range v{a->v, N * H * a->dv * es}, la{a->log_alpha, N * H * (gate_head ? 1 : a->dk) * 4};
  const Range be{a->beta, N * H * 4}, cu{a->cu_seqlens, 4 * ((size_t)a->num_seqs + 1)};
  const Range mk{a->pad_mask, a->pad_mask ? N : 0};
  const size_t sbytes = (size_t)a->num_seqs * H * a->dk * a->dv * 4;
  const Range s0{a->init_state, a->init_state ? sbytes : 0};
  const Range s1{a->final_state, a->final_state ? sbytes : 0};
  const Range o{a->o, N * H * a->dv * es};
  const Range ws{a->workspace, a->workspace ? a->workspace_bytes : 0};
  if (N > 0 && (!a->q || !a->k || !a->v || !a->log_alpha || !a->beta || !a->o))
    return KDA_ERR_INVALID_ARG;
  const void *need16[] = {a->q, a->k, a->v, gate_head ? nullptr : (const void *)a->log_alpha, a->o,
                          (const void *)a->init_state, (const void *)a->final_state};
  for (const void *p : need16)
    if (p && !aligned(p, 16)) return KDA_ERR_INVALID_ARG;
  if (!aligned(a->beta, 4) || !aligned(a->cu_seqlens, 4) || !aligned(a->log_alpha, 4))
    return KDA_ERR_INVALID_ARG;
  // A pad mask needs at least the span table; a larger workspace (up to
  // kda_prefill_workspace_size) only selects a faster path.
  if (a->pad_mask && (!a->workspace || a->workspace_bytes < spans_bytes(a->num_seqs)))
    return KDA_ERR_INVALID_ARG;
  if (a->workspace && !aligned(a->workspace, 256)) return KDA_ERR_INVALID_ARG;
  // o and final_state must not overlap any input; init/final may coincide exactly
  const Range inputs[] = {q, k, v, la, be, cu, mk, s0, ws};
  for (const Range &r : inputs) {
    if (overlap(o, r)) return KDA_ERR_INVALID_ARG;
    if (overlap(s1, r) && !(r.p == s0.p && s1.p == s0.p)) return KDA_ERR_INVALID_ARG;
  }
  if (overlap(o, s1)) return KDA_ERR_INVALID_ARG;
  if (overlap(ws, q) || overlap(ws, k) || overlap(ws, v) || overlap(ws, la) || overlap(ws, be) ||
      overlap(ws, cu) || overlap(ws, mk) || overlap(ws, s0))
    return KDA_ERR_INVALID_ARG;

  unsigned *err = nullptr, *site = nullptr;
  if (error_word(&err) != KDA_OK || timeout_site_word(&site) != KDA_OK) return KDA_ERR_CUDA;
  PrefillParams p;
  p.num_seqs = a->num_seqs;
  p.N = a->total_tokens;
  p.H = a->H;
  p.dk = a->dk;
  p.dv = a->dv;
  p.chunk = chunk;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.log_alpha = a->log_alpha;
  p.beta = a->beta;
  p.cu = a->cu_seqlens;
  p.mask = a->pad_mask;
  p.init_state = a->init_state;
  p.o = a->o;
  p.final_state = a->final_state;
  p.err = err;
  p.gate_head = gate_head ? 1 : 0;
  p.wait_cycles = g_wait_cycles.load(std::memory_order_relaxed);
  p.fault = g_fault.load(std::memory_order_relaxed);
  p.site = site;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf16 = a->dtype == KDA_BF16;
  p.spans = nullptr;
  // Two-kernel path when the workspace holds the per-chunk items; otherwise the
  // fused tensor-core kernel (or the CUDA-core kernel for other shapes).
  // Chunks of 128 / 256 rows exist only on the workspace-backed tensor-core path.
  if (big && (!a->workspace || a->workspace_bytes < prefill_bigchunk_workspace(a->total_tokens, a->num_seqs,
                                                                                 a->H, chunk)))
    return KDA_ERR_UNSUPPORTED;
  const bool split = prefill_split_supported(p, bf16) && a->workspace &&
                     a->workspace_bytes >= prefill_split_workspace(a->total_tokens, a->num_seqs, a->H);
  SeqSpan *spans = (big || split || a->pad_mask) ? static_cast<SeqSpan *>(a->workspace) : nullptr;
  if (launch_prefill_prepass(p, bf16, spans, s) != cudaSuccess) return KDA_ERR_CUDA;
  p.spans = spans;
  cudaError_t e;
  if (big) e = launch_prefill_bigchunk(p, spans, a->workspace, s);
  else if (split) e = launch_prefill_split(p, spans, a->workspace, s);
  else if (prefill_tc_supported(p, bf16)) e = launch_prefill_tc(p, s);
  else e = launch_prefill_simt(p, bf16, s);
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_decode(const kda_decode_args *a, void *stream) {
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->dtype != KDA_F32 && a->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 1 || a->dk <= 0 || a->dv <= 0) return KDA_ERR_INVALID_ARG;
  if (a->gate != KDA_GATE_CHANNEL && a->gate != KDA_GATE_HEAD) return KDA_ERR_INVALID_ARG;
  const bool gate_head = a->gate == KDA_GATE_HEAD;
  if (!head_dim_ok(a->dk) || !head_dim_ok(a->dv)) return KDA_ERR_UNSUPPORTED;
  if (a->B == 0) return KDA_OK;
  if (!a->q || !a->k || !a->v || !a->log_alpha || !a->beta || !a->state || !a->o)
    return KDA_ERR_INVALID_ARG;
  const size_t B = (size_t)a->B, H = (size_t)a->H, es = elem_bytes(a->dtype);
  const Range q{a->q, B * H * a->dk * es}, k{a->k, B * H * a->dk * es};
  const Range v{a->v, B * H * a->dv * es}, la{a->log_alpha, B * H * (gate_head ? 1 : a->dk) * 4};
  const Range be{a->beta, B * H * 4}, mk{a->mask, a->mask ? B : 0};
  const Range st{a->state, B * H * a->dk * a->dv * 4}, o{a->o, B * H * a->dv * es};
  if (!aligned(a->state, 16) || !aligned(a->beta, 4) || !aligned(a->log_alpha, 4))
    return KDA_ERR_INVALID_ARG;
  if (!aligned(a->q, es) || !aligned(a->k, es) || !aligned(a->v, es) || !aligned(a->o, es))
    return KDA_ERR_INVALID_ARG;
  const Range others[] = {q, k, v, la, be, mk};
  for (const Range &r : others)
    if (overlap(o, r) || overlap(st, r)) return KDA_ERR_INVALID_ARG;
  if (overlap(o, st)) return KDA_ERR_INVALID_ARG;
  unsigned *err = nullptr;
  if (error_word(&err) != KDA_OK) return KDA_ERR_CUDA;
  DecodeParams p;
  p.B = a->B;
  p.H = a->H;
  p.dk = a->dk;
  p.dv = a->dv;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.log_alpha = a->log_alpha;
  p.beta = a->beta;
  p.mask = a->mask;
  p.state = a->state;
  p.o = a->o;
  p.err = err;
  p.gate_head = gate_head ? 1 : 0;
  return launch_decode(p, a->dtype == KDA_BF16, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_short_conv(const kda_conv_args *a, void *stream) {
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->dtype != KDA_F32 && a->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (a->num_seqs < 0 || a->total_tokens < 0 || a->D < 8 || a->D % 8 != 0) return KDA_ERR_INVALID_ARG;
  if (a->width < 1 || a->width > 4) return KDA_ERR_UNSUPPORTED;
  if (a->num_seqs == 0) return a->total_tokens == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
  if (!a->cu_seqlens || !a->weight) return KDA_ERR_INVALID_ARG;
  if (a->total_tokens > 0 && (!a->x || !a->y)) return KDA_ERR_INVALID_ARG;
  const size_t N = (size_t)a->total_tokens, D = (size_t)a->D, es = elem_bytes(a->dtype);
  const size_t sbytes = (size_t)a->num_seqs * (a->width - 1) * D * 4;
  const Range x{a->x, N * D * es}, y{a->y, N * D * es}, w{a->weight, D * a->width * 4};
  const Range bi{a->bias, a->bias ? D * 4 : 0}, cu{a->cu_seqlens, 4 * ((size_t)a->num_seqs + 1)};
  const Range mk{a->pad_mask, a->pad_mask ? N : 0};
  const Range s0{a->state_in, a->state_in ? sbytes : 0}, s1{a->state_out, a->state_out ? sbytes : 0};
  if ((a->x && !aligned(a->x, 16)) || (a->y && !aligned(a->y, 16)) || !aligned(a->weight, 4) ||
      !aligned(a->bias, 4) || !aligned(a->cu_seqlens, 4) || !aligned(a->state_in, 16) ||
      !aligned(a->state_out, 4))
    return KDA_ERR_INVALID_ARG;
  const Range inputs[] = {x, w, bi, cu, mk, s0};
  for (const Range &r : inputs) {
    if (overlap(y, r)) return KDA_ERR_INVALID_ARG;
    if (overlap(s1, r) && !(r.p == s0.p && s1.p == s0.p)) return KDA_ERR_INVALID_ARG;
  }
  if (overlap(y, s1)) return KDA_ERR_INVALID_ARG;
  unsigned *err = nullptr;
  if (error_word(&err) != KDA_OK) return KDA_ERR_CUDA;
  ConvParams p;
  p.num_seqs = a->num_seqs;
  p.N = a->total_tokens;
  p.D = a->D;
  p.W = a->width;
  p.x = a->x;
  p.weight = a->weight;
  p.bias = a->bias;
  p.cu = a->cu_seqlens;
  p.mask = a->pad_mask;
  p.state_in = a->state_in;
  p.state_out = a->state_out;
  p.y = a->y;
  p.err = err;
  return launch_short_conv(p, a->dtype == KDA_BF16, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_prefill_backward_workspace_size(const kda_backward_args *a) {
  if (!a || a->total_tokens < 0 || a->num_seqs < 0 || a->H < 1 || a->dk <= 0 || a->dv <= 0) return 0;
  return backward_workspace(a->total_tokens, a->num_seqs, a->H, a->dk, a->dv);
}

kda_status kda_prefill_backward(const kda_backward_args *a, void *stream) {
  if (!a) return KDA_ERR_INVALID_ARG;
  if (a->dtype != KDA_F32 && a->dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (a->num_seqs < 0 || a->total_tokens < 0 || a->H < 1 || a->dk <= 0 || a->dv <= 0)
    return KDA_ERR_INVALID_ARG;
  if (!head_dim_ok(a->dk) || !head_dim_ok(a->dv)) return KDA_ERR_UNSUPPORTED;
  if (a->gate != KDA_GATE_CHANNEL && a->gate != KDA_GATE_HEAD) return KDA_ERR_INVALID_ARG;
  const bool gate_head = a->gate == KDA_GATE_HEAD;
  if (a->num_seqs == 0) return a->total_tokens == 0 ? KDA_OK : KDA_ERR_INVALID_ARG;
  if (!a->cu_seqlens) return KDA_ERR_INVALID_ARG;
  const size_t N = (size_t)a->total_tokens, H = (size_t)a->H, es = elem_bytes(a->dtype);
  const size_t dk = a->dk, dv = a->dv, lad = gate_head ? 1 : dk;
  const size_t sbytes = (size_t)a->num_seqs * H * dk * dv * 4;
  if (N > 0 && (!a->q || !a->k || !a->v || !a->log_alpha || !a->beta || !a->grad_o || !a->grad_q ||
                !a->grad_k || !a->grad_v || !a->grad_log_alpha || !a->grad_beta))
    return KDA_ERR_INVALID_ARG;
  if (N > 0 && (!a->workspace ||
                a->workspace_bytes < backward_workspace(a->total_tokens, a->num_seqs, a->H, a->dk, a->dv)))
    return KDA_ERR_INVALID_ARG;
  const Range q{a->q, N * H * dk * es}, k{a->k, N * H * dk * es}, v{a->v, N * H * dv * es};
  const Range la{a->log_alpha, N * H * lad * 4}, be{a->beta, N * H * 4};
  const Range cu{a->cu_seqlens, 4 * ((size_t)a->num_seqs + 1)}, mk{a->pad_mask, a->pad_mask ? N : 0};
  const Range s0{a->init_state, a->init_state ? sbytes : 0};
  const Range go{a->grad_o, N * H * dv * 4}, gf{a->grad_final_state, a->grad_final_state ? sbytes : 0};
  const Range ws{a->workspace, a->workspace ? a->workspace_bytes : 0};
  const Range outs[] = {{a->grad_q, N * H * dk * 4}, {a->grad_k, N * H * dk * 4}, {a->grad_v, N * H * dv * 4},
                        {a->grad_log_alpha, N * H * lad * 4}, {a->grad_beta, N * H * 4},
                        {a->grad_init_state, a->grad_init_state ? sbytes : 0}, ws};
  const Range ins[] = {q, k, v, la, be, cu, mk, s0, go, gf};
  for (int i = 0; i < 7; ++i) {
    for (const Range &r : ins)
      if (overlap(outs[i], r)) return KDA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 7; ++j)
      if (overlap(outs[i], outs[j])) return KDA_ERR_INVALID_ARG;
  }
  const void *need16[] = {a->q, a->k, a->v, a->grad_o, a->grad_q, a->grad_k, a->grad_v, a->init_state,
                          a->grad_final_state, a->grad_init_state};
  for (const void *p : need16)
    if (p && !aligned(p, 16)) return KDA_ERR_INVALID_ARG;
  if (!aligned(a->log_alpha, 4) || !aligned(a->beta, 4) || !aligned(a->grad_log_alpha, 4) ||
      !aligned(a->grad_beta, 4) || !aligned(a->cu_seqlens, 4) || (a->workspace && !aligned(a->workspace, 256)))
    return KDA_ERR_INVALID_ARG;
  unsigned *err = nullptr;
  if (error_word(&err) != KDA_OK) return KDA_ERR_CUDA;
  BackwardParams p;
  p.num_seqs = a->num_seqs;
  p.N = a->total_tokens;
  p.H = a->H;
  p.dk = a->dk;
  p.dv = a->dv;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.log_alpha = a->log_alpha;
  p.beta = a->beta;
  p.cu = a->cu_seqlens;
  p.mask = a->pad_mask;
  p.init_state = a->init_state;
  p.d_o = a->grad_o;
  p.d_final_state = a->grad_final_state;
  p.gq = a->grad_q;
  p.gk = a->grad_k;
  p.gv = a->grad_v;
  p.gla = a->grad_log_alpha;
  p.gbeta = a->grad_beta;
  p.g_init_state = a->grad_init_state;
  p.ws = static_cast<float *>(a->workspace);
  p.err = err;
  p.gate_head = gate_head ? 1 : 0;
  return launch_backward(p, a->dtype == KDA_BF16, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_debug_set_fault(int fault, long long wait_cycles) {
  if (fault & ~FAULT_STARVE_STATE_LOADS) return KDA_ERR_INVALID_ARG;
  g_fault.store(fault, std::memory_order_relaxed);
  g_wait_cycles.store(wait_cycles > 0 ? wait_cycles : kDefaultWaitCycles, std::memory_order_relaxed);
  return KDA_OK;
}

int kda_debug_timeout_site(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return -1;
  unsigned *site = nullptr;
  if (timeout_site_word(&site) != KDA_OK) return -1;
  unsigned code = 0;
  if (cudaMemcpy(&code, site, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  const unsigned zero = 0;
  if (code != 0 && cudaMemcpy(site, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return -1;
  return (int)code;
}

kda_status kda_get_device_status(void *stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KDA_ERR_CUDA;
  unsigned *err = nullptr;
  if (error_word(&err) != KDA_OK) return KDA_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return KDA_ERR_CUDA;
  if (word == 0) return KDA_OK;
  const unsigned zero = 0;
  if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return KDA_ERR_CUDA;
  if (word & ERR_BIT_TIMEOUT) return KDA_ERR_DEVICE_TIMEOUT;
  return KDA_ERR_DEVICE_CHECK;
}

}  // extern "C"
