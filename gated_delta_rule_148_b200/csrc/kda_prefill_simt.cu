// KDA chunkwise prefill on CUDA cores (fp32 arithmetic throughout).
//
// This is the fp32 path (fp32 q/k/v; tolerance class 1e-4) and the general
// path for shapes the tensor-core kernel is not built for.  It computes the
// chunkwise WY/UT form of the recurrence ("Kimi Linear's 75% KV cache cut
// ...", theclarity.today, fourth paragraph: chunks plus the WY representation
// turn a chunk's rank-1 updates into a triangular solve and dense products;
// "Kimi Linear wlasnie pokonal ...", remio.ai: blockwise algorithm with a
// diagonal-plus-low-rank transition).  Per chunk of C positions with incoming
// state S0, g = inclusive per-channel cumsum of log_alpha in the chunk:
//   A[r,i] = beta_r sum_c k[r,c] k[i,c] e^{g[r,c]-g[i,c]}   (i < r)
//   M[r,i] =        sum_c q[r,c] k[i,c] e^{g[r,c]-g[i,c]}   (i <= r)
//   T = (I + A)^{-1};  W = T (beta K e^g);  U_v = T (beta V)
//   U = U_v - W S0;  O = (Q e^g) S0 + M U;
//   S = Diag(e^{g_last}) S0 + (K e^{g_last - g})^T U.
// Every exponent here is <= 0 (g is non-increasing along the chunk), so the
// path is exact-safe for any log_alpha <= 0.  One CTA owns one (sequence,
// head, 32-column slice of d_v) and walks its chunks in order; the state
// slice stays in shared memory for the whole sequence.
#include <climits>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kDvTile = 32;

template <int DK, int C>
struct SimtSmem {
  static constexpr int KS = DK + 1;       // padded row stride of [C][DK] tiles
  static constexpr int CS = C + 1;        // padded row stride of [C][C] tiles
  static constexpr int VS = kDvTile + 1;  // padded row stride of [*][dv tile] tiles
  static constexpr int kK = 0;                     // K, then K e^{g_last - g}
  static constexpr int kQ = kK + C * KS;           // Q, then Q e^g
  static constexpr int kG = kQ + C * KS;           // g, then W
  static constexpr int kWr = kG + C * KS;          // beta K e^g
  static constexpr int kA = kWr + C * KS;          // A
  static constexpr int kM = kA + C * CS;           // M
  static constexpr int kT = kM + C * CS;           // T
  static constexpr int kV = kT + C * CS;           // beta V
  static constexpr int kU = kV + C * VS;           // U_v, then U
  static constexpr int kS = kU + C * VS;           // state slice [DK][dv tile]
  static constexpr int kB = kS + DK * VS;          // beta [C]
  static constexpr int kGe = kB + C;               // g_last [DK]
  static constexpr int kFloats = kGe + DK;
  static constexpr size_t kBytes = sizeof(float) * (size_t)kFloats;
};

// Span of a sequence: [begin, end) packed rows actually processed.
__device__ __forceinline__ SeqSpan get_span(const PrefillParams &p, int b) {
  if (p.spans) return p.spans[b];
  SeqSpan s;
  s.seq_begin = p.cu[b];
  s.begin = p.cu[b];
  s.end = p.cu[b + 1];
  s.pad_inside = 0;
  return s;
}

template <int DK, int C, bool BF16>
__global__ void __launch_bounds__(kThreads)
prefill_simt_kernel(PrefillParams p) {
  using L = SimtSmem<DK, C>;
  extern __shared__ float sm[];
  float *Ks = sm + L::kK, *Qs = sm + L::kQ, *Gs = sm + L::kG, *Wr = sm + L::kWr;
  float *As = sm + L::kA, *Ms = sm + L::kM, *Ts = sm + L::kT, *Vs = sm + L::kV;
  float *Us = sm + L::kU, *Ss = sm + L::kS, *Bs = sm + L::kB, *Ge = sm + L::kGe;
  constexpr int KS = L::KS, CS = L::CS, VS = L::VS;

  if (device_error_latched(p.err)) return;
  const int tiles = p.dv / kDvTile;
  const int tile = blockIdx.x % tiles;
  const int h = (blockIdx.x / tiles) % p.H;
  const int b = blockIdx.x / (tiles * p.H);
  const int tid = threadIdx.x;
  const int dv0 = tile * kDvTile;
  const int H = p.H, DV = p.dv;
  const SeqSpan span = get_span(p, b);

  // initial state slice
  for (int e = tid; e < DK * kDvTile; e += kThreads) {
    const int c = e / kDvTile, j = e % kDvTile;
    Ss[c * VS + j] = p.init_state
        ? p.init_state[(((size_t)b * H + h) * DK + c) * DV + dv0 + j] : 0.f;
  }

  for (int c0 = span.begin; c0 < span.end; c0 += C) {
    __syncthreads();
    // ---- load the chunk; tail rows and pads become identity steps
    for (int e = tid; e < C * DK; e += kThreads) {
      const int r = e / DK, c = e % DK;
      const int pos = c0 + r;
      const bool ok = pos < span.end && (p.mask == nullptr || p.mask[pos] != 0);
      const size_t gi = ((size_t)pos * H + h) * DK + c;
      Ks[r * KS + c] = ok ? load_elem<BF16>(p.k, gi) : 0.f;
      Qs[r * KS + c] = ok ? load_elem<BF16>(p.q, gi) : 0.f;
      Gs[r * KS + c] = ok ? p.log_alpha[la_index(pos, h, H, DK, c, p.gate_head)] : 0.f;
    }
    for (int e = tid; e < C * kDvTile; e += kThreads) {
      const int r = e / kDvTile, j = e % kDvTile;
      const int pos = c0 + r;
      const bool ok = pos < span.end && (p.mask == nullptr || p.mask[pos] != 0);
      Vs[r * VS + j] = ok ? load_elem<BF16>(p.v, ((size_t)pos * H + h) * DV + dv0 + j) : 0.f;
    }
    for (int r = tid; r < C; r += kThreads) {
      const int pos = c0 + r;
      const bool ok = pos < span.end && (p.mask == nullptr || p.mask[pos] != 0);
      Bs[r] = ok ? p.beta[(size_t)pos * H + h] : 0.f;
    }
    __syncthreads();
    // ---- g: inclusive per-channel cumsum over the chunk
    for (int c = tid; c < DK; c += kThreads) {
      float acc = 0.f;
      for (int r = 0; r < C; ++r) {
        acc += Gs[r * KS + c];
        Gs[r * KS + c] = acc;
      }
      Ge[c] = acc;
    }
    __syncthreads();
    // ---- A and M (decay applied per element; all exponents <= 0)
    for (int e = tid; e < C * C; e += kThreads) {
      const int r = e / C, i = e % C;
      float a = 0.f, m = 0.f;
      if (i <= r) {
        for (int c = 0; c < DK; ++c) {
          const float d = __expf(Gs[r * KS + c] - Gs[i * KS + c]);
          const float kd = Ks[i * KS + c] * d;
          a = fmaf(Ks[r * KS + c], kd, a);
          m = fmaf(Qs[r * KS + c], kd, m);
        }
      }
      As[r * CS + i] = (i < r) ? Bs[r] * a : 0.f;
      Ms[r * CS + i] = (i <= r) ? m : 0.f;
    }
    __syncthreads();
    // ---- operand transforms
    for (int e = tid; e < C * DK; e += kThreads) {
      const int r = e / DK, c = e % DK;
      const float g = Gs[r * KS + c];
      const float eg = __expf(g);
      const float kk = Ks[r * KS + c];
      Wr[r * KS + c] = Bs[r] * kk * eg;
      Qs[r * KS + c] *= eg;
      Ks[r * KS + c] = kk * __expf(Ge[c] - g);
    }
    for (int e = tid; e < C * kDvTile; e += kThreads) {
      const int r = e / kDvTile, j = e % kDvTile;
      Vs[r * VS + j] *= Bs[r];
    }
    // ---- T = (I + A)^{-1}: forward substitution, one column per thread
    for (int j = tid; j < C; j += kThreads) {
      for (int r = 0; r < C; ++r) {
        float t;
        if (r < j) t = 0.f;
        else if (r == j) t = 1.f;
        else {
          t = 0.f;
          for (int i = j; i < r; ++i) t = fmaf(As[r * CS + i], Ts[i * CS + j], t);
          t = -t;
        }
        Ts[r * CS + j] = t;
      }
    }
    __syncthreads();
    // ---- W = T Wr (into the g buffer), U_v = T (beta V)
    for (int e = tid; e < C * DK; e += kThreads) {
      const int r = e / DK, c = e % DK;
      float acc = 0.f;
      for (int i = 0; i <= r; ++i) acc = fmaf(Ts[r * CS + i], Wr[i * KS + c], acc);
      Gs[r * KS + c] = acc;
    }
    for (int e = tid; e < C * kDvTile; e += kThreads) {
      const int r = e / kDvTile, j = e % kDvTile;
      float acc = 0.f;
      for (int i = 0; i <= r; ++i) acc = fmaf(Ts[r * CS + i], Vs[i * VS + j], acc);
      Us[r * VS + j] = acc;
    }
    __syncthreads();
    // ---- state-dependent part: U = U_v - W S
    for (int e = tid; e < C * kDvTile; e += kThreads) {
      const int r = e / kDvTile, j = e % kDvTile;
      float acc = 0.f;
      for (int c = 0; c < DK; ++c) acc = fmaf(Gs[r * KS + c], Ss[c * VS + j], acc);
      Us[r * VS + j] -= acc;
    }
    __syncthreads();
    // ---- O = (Q e^g) S + M U
    for (int e = tid; e < C * kDvTile; e += kThreads) {
      const int r = e / kDvTile, j = e % kDvTile;
      const int pos = c0 + r;
      if (pos >= span.end) continue;
      float acc = 0.f;
      for (int c = 0; c < DK; ++c) acc = fmaf(Qs[r * KS + c], Ss[c * VS + j], acc);
      for (int i = 0; i <= r; ++i) acc = fmaf(Ms[r * CS + i], Us[i * VS + j], acc);
      const bool ok = p.mask == nullptr || p.mask[pos] != 0;
      store_elem<BF16>(p.o, ((size_t)pos * H + h) * DV + dv0 + j, ok ? acc : 0.f);
    }
    __syncthreads();
    // ---- S = Diag(e^{g_last}) S + (K e^{g_last - g})^T U
    for (int e = tid; e < DK * kDvTile; e += kThreads) {
      const int c = e / kDvTile, j = e % kDvTile;
      float acc = __expf(Ge[c]) * Ss[c * VS + j];
      for (int i = 0; i < C; ++i) acc = fmaf(Ks[i * KS + c], Us[i * VS + j], acc);
      Ss[c * VS + j] = acc;
    }
  }
  __syncthreads();
  if (p.final_state) {
    for (int e = tid; e < DK * kDvTile; e += kThreads) {
      const int c = e / kDvTile, j = e % kDvTile;
      p.final_state[(((size_t)b * H + h) * DK + c) * DV + dv0 + j] = Ss[c * VS + j];
    }
  }
}

template <int DK, int C>
cudaError_t launch_dk_c(const PrefillParams &p, bool bf16, cudaStream_t s) {
  using L = SimtSmem<DK, C>;
  const unsigned grid = (unsigned)p.num_seqs * p.H * (p.dv / kDvTile);
  cudaError_t e;
  if (bf16) {
    e = cudaFuncSetAttribute(prefill_simt_kernel<DK, C, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (e != cudaSuccess) return e;
    prefill_simt_kernel<DK, C, true><<<grid, kThreads, L::kBytes, s>>>(p);
  } else {
    e = cudaFuncSetAttribute(prefill_simt_kernel<DK, C, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (e != cudaSuccess) return e;
    prefill_simt_kernel<DK, C, false><<<grid, kThreads, L::kBytes, s>>>(p);
  }
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dk(const PrefillParams &p, bool bf16, cudaStream_t s) {
  switch (p.chunk) {
    case 16: return launch_dk_c<DK, 16>(p, bf16, s);
    case 32: return launch_dk_c<DK, 32>(p, bf16, s);
    case 64: return launch_dk_c<DK, 64>(p, bf16, s);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------- pre-pass
// Checks cu_seqlens (every block checks the whole array, block 0 latches the
// error) and, with a pad mask, computes each sequence's span of valid
// positions and writes o = 0 at every pad position of the sequence.
template <bool BF16>
__global__ void __launch_bounds__(256)
prefill_prepass_kernel(PrefillParams p, SeqSpan *spans) {
  __shared__ int s_bad, s_first, s_last, s_count;
  const int tid = threadIdx.x;
  if (tid == 0) { s_bad = 0; s_first = INT_MAX; s_last = -1; s_count = 0; }
  __syncthreads();
  if (device_error_latched(p.err)) return;
  int bad = 0;
  for (int i = tid; i <= p.num_seqs; i += blockDim.x) {
    const int v = p.cu[i];
    if (v < 0 || v > p.N) bad = 1;
    if (i == 0 && v != 0) bad = 1;
    if (i == p.num_seqs && v != p.N) bad = 1;
    if (i > 0 && p.cu[i - 1] > v) bad = 1;
  }
  if (bad) atomicOr(&s_bad, 1);
  __syncthreads();
  if (s_bad) {
    if (blockIdx.x == 0 && tid == 0) atomicOr(p.err, ERR_BIT_CHECK);
    return;
  }
  if (spans == nullptr) return;
  const int b = blockIdx.x;
  const int beg = p.cu[b], end = p.cu[b + 1];
  if (p.mask == nullptr) {      // no pads: the span is the whole sequence
    if (tid == 0) {
      SeqSpan sp;
      sp.seq_begin = beg;
      sp.begin = beg;
      sp.end = end;
      sp.pad_inside = 0;
      spans[b] = sp;
    }
    return;
  }
  int first = INT_MAX, last = -1, count = 0;
  for (int pos = beg + tid; pos < end; pos += blockDim.x) {
    if (p.mask[pos]) {
      first = min(first, pos);
      last = max(last, pos);
      ++count;
    }
  }
  atomicMin(&s_first, first);
  atomicMax(&s_last, last);
  atomicAdd(&s_count, count);
  __syncthreads();
  // zero o at every pad position of this sequence: one warp per position
  const int row = p.H * p.dv;
  const int lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  for (int pos = beg + warp; pos < end; pos += nwarps) {
    if (p.mask[pos]) continue;
    for (int e = lane; e < row; e += 32) store_elem<BF16>(p.o, (size_t)pos * row + e, 0.f);
  }
  if (tid == 0) {
    SeqSpan sp;
    sp.seq_begin = beg;
    if (s_count == 0) {
      sp.begin = beg;
      sp.end = beg;
      sp.pad_inside = 0;
    } else {
      sp.begin = s_first;
      sp.end = s_last + 1;
      sp.pad_inside = (s_count != s_last + 1 - s_first) ? 1 : 0;
    }
    spans[b] = sp;
  }
}

}  // namespace

cudaError_t launch_prefill_prepass(const PrefillParams &p, bool bf16, SeqSpan *spans,
                                   cudaStream_t s) {
  const unsigned grid = (p.num_seqs > 0 && spans) ? (unsigned)p.num_seqs : 1u;
  if (bf16) prefill_prepass_kernel<true><<<grid, 256, 0, s>>>(p, spans);
  else prefill_prepass_kernel<false><<<grid, 256, 0, s>>>(p, spans);
  return cudaGetLastError();
}

cudaError_t launch_prefill_simt(const PrefillParams &p, bool bf16, cudaStream_t s) {
  if (p.num_seqs == 0) return cudaSuccess;
  if (p.dv % kDvTile != 0) return cudaErrorInvalidValue;
  if (p.dk == 128) return launch_dk<128>(p, bf16, s);
  if (p.dk == 64) return launch_dk<64>(p, bf16, s);
  return cudaErrorInvalidValue;
}

}  // namespace kda
