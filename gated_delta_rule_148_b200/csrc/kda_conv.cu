// Padding-correct short causal convolution with a carried convolution state.
//
// Per sequence and channel c, over the sequence's VALID positions only (a pad
// neither enters the window nor moves it, and its output is 0):
//   y_t[c] = bias[c] + sum_{i<W} weight[c][i] * u_i[c],
// u_0 .. u_{W-1} = the W-1 valid inputs before t (oldest first) followed by x_t;
// before the sequence's first valid inputs the window holds conv_state (W-1
// rows, oldest first; zeros when none is given).  The final window (last W-1
// valid inputs, completed from the old state when the sequence is short)
// becomes the new conv_state.  ("Transformers Community Reports Kimi Linear
// Cache Bug", ainews: padded entries must not enter the convolution window, nor
// advance the convolution state, of a cached continuation.)
//
// Layout: x, y [N, D] (bf16 or fp32), weight [D, W] fp32, bias [D] fp32,
// conv_state [B, W-1, D] fp32.  The operation is HBM-bound (read x, write y):
// kernel A gives each CTA a contiguous span of packed positions (about N / (2 x SMs
// per channel block): one wave) and up to 2048 channels; the pad mask of the span
// is compacted once (warp ballots, 256 positions a pass) into the list of valid
// rows, and each thread walks those rows for its 8 consecutive channels with the
// window in registers and the next 8 rows' loads already in flight (a ring of raw
// 16- or 32-byte loads), so each thread keeps 8 loads outstanding and fills its
// ring once per span.  Kernel B writes the new
// state after kernel A, one thread per (sequence, channel), so conv_state may be
// updated in place.
#include "kda_internal.cuh"

namespace kda {
namespace conv {

constexpr int kSeg = 256;            // packed positions per compaction pass (one per thread)
constexpr int kMaxSpan = 4096;       // packed positions per CTA at most (the list of valid rows)
constexpr int kThreads = 256;
constexpr int kPer = 8;              // channels per thread
constexpr int kChan = kPer * kThreads;  // channels per CTA
constexpr int kRing = 8;             // rows whose loads are in flight ahead of the walk (bf16)
constexpr int kMaxW = 4;
static_assert(kSeg == kThreads, "one compaction ballot per position");

// Source of a window entry: a packed position (>= 0) or state row j (encoded -1 - j).
struct Hist {
  int src[kMaxW - 1];
};

// The W-1 newest valid positions of sequence [sb, before) (oldest first); entries the
// sequence cannot fill come from the newest state rows.  Scans the mask backwards.
__device__ __forceinline__ Hist history_before(const uint8_t *mask, int sb, int before, int W) {
  Hist hs;
  const int need = W - 1;
  int found = 0;
  int tmp[kMaxW - 1];
  for (int pos = before - 1; pos >= sb && found < need; --pos)
    if (mask == nullptr || mask[pos] != 0) tmp[found++] = pos;
  // tmp[0] is the newest; entry need-1-f of the window is tmp[f]
#pragma unroll
  for (int j = 0; j < kMaxW - 1; ++j) {
    if (j >= need) break;
    const int f = need - 1 - j;          // how many newer entries follow slot j
    if (f < found) hs.src[j] = tmp[f];
    else hs.src[j] = -1 - (j + found);   // state row: slots not filled by the sequence
  }
  return hs;
}

// Raw loads of kPer consecutive channels of one row (kPer bf16 = kPer / 2 words, or
// kPer fp32 words), unpacked separately so that several rows' loads can be in flight.
template <bool BF16> __host__ __device__ constexpr int raw_words() { return BF16 ? kPer / 2 : kPer; }
static_assert(kPer == 2 || kPer == 4 || kPer == 8, "row loads of 4 to 32 bytes");
template <bool BF16> struct RawRow { uint32_t w[raw_words<BF16>()]; };

template <bool BF16>
__device__ __forceinline__ RawRow<BF16> load_row(const void *x, size_t row, int D, int c) {
  constexpr int n = raw_words<BF16>();
  const uint32_t *src = reinterpret_cast<const uint32_t *>(x) + (row * D + c) * (BF16 ? 1 : 2) / 2;
  RawRow<BF16> r;
  if constexpr (n % 4 == 0) {
#pragma unroll
    for (int e = 0; e < n; e += 4) {
      const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src) + e / 4);
      r.w[e] = u.x; r.w[e + 1] = u.y; r.w[e + 2] = u.z; r.w[e + 3] = u.w;
    }
  } else if constexpr (n == 2) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(src));
    r.w[0] = u.x; r.w[1] = u.y;
  } else {
    r.w[0] = __ldg(src);
  }
  return r;
}

template <bool BF16>
__device__ __forceinline__ void unpack_row(const RawRow<BF16> &r, float *v) {
  if constexpr (BF16) {
#pragma unroll
    for (int e = 0; e < kPer / 2; ++e) {
      v[2 * e] = __uint_as_float(r.w[e] << 16);
      v[2 * e + 1] = __uint_as_float(r.w[e] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) v[e] = __uint_as_float(r.w[e]);
  }
}

// Two fp32 -> packed bf16x2, round to nearest even; `lo` lands in the low half.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

template <bool BF16>
__device__ __forceinline__ void store_row(void *y, size_t row, int D, int c, const float *v) {
  RawRow<BF16> r;
  if constexpr (BF16) {
#pragma unroll
    for (int e = 0; e < kPer / 2; ++e) r.w[e] = bf16x2_rn(v[2 * e], v[2 * e + 1]);
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) r.w[e] = __float_as_uint(v[e]);
  }
  constexpr int n = raw_words<BF16>();
  uint32_t *dst = reinterpret_cast<uint32_t *>(y) + (row * D + c) * (BF16 ? 1 : 2) / 2;
  if constexpr (n % 4 == 0) {
#pragma unroll
    for (int e = 0; e < n; e += 4)
      reinterpret_cast<uint4 *>(dst)[e / 4] = make_uint4(r.w[e], r.w[e + 1], r.w[e + 2], r.w[e + 3]);
  } else if constexpr (n == 2) {
    *reinterpret_cast<uint2 *>(dst) = make_uint2(r.w[0], r.w[1]);
  } else {
    *dst = r.w[0];
  }
}

// Kernel A: outputs of packed positions [span*blockIdx.x, +span), channels
// [kChan*blockIdx.y, +kChan), span chosen on the host so that the grid is about
// one wave (every CTA then fills its load ring once, not once per short block).
// Thread t owns channels 8t .. 8t+7 and walks the CTA's valid rows in order with
// the window in registers, so each x row is read once; the loads of one row are
// coalesced across the CTA's threads, and the ring keeps the loads of the next
// kRing rows in flight.
template <bool BF16, int KW>      // KW: the window width W (1..4), fixed at compile time
__global__ void __launch_bounds__(kThreads, 2) conv_kernel(ConvParams p, int span) {
  __shared__ int vpos[kMaxSpan];
  __shared__ int wcnt[kThreads / 32];
  __shared__ Hist hist_sh;
  if (device_error_latched(p.err)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int W = KW;
  const int D = p.D, B = p.num_seqs;
  const int s0 = blockIdx.x * span, s1 = min(s0 + span, p.N);
  const int c_lo = blockIdx.y * kChan, nch = min(kChan, D - c_lo);
  if (blockIdx.x == 0 && blockIdx.y == 0) {       // cu_seqlens: 0, non-decreasing, ends at N
    bool bad = false;
    for (int b = tid; b < B; b += kThreads) bad |= p.cu[b] > p.cu[b + 1];
    if (tid == 0) bad |= p.cu[0] != 0 || p.cu[B] != p.N;
    if (bad) atomicOr(p.err, ERR_BIT_CHECK);
  }
  // this thread's channels and their taps
  const int cl = tid * kPer, c = c_lo + cl;
  const bool mine = cl < nch;
  float wt[kMaxW - 1][kPer], wx[kPer], bz[kPer];      // window taps, the current row's tap, bias
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    bz[j] = (mine && p.bias) ? p.bias[c + j] : 0.f;
    wx[j] = mine ? p.weight[(size_t)(c + j) * W + (W - 1)] : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxW - 1; ++i)
      wt[i][j] = (mine && i < W - 1) ? p.weight[(size_t)(c + j) * W + i] : 0.f;
  }
  // first sequence with cu[b + 1] > s0
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (p.cu[mid + 1] <= s0) lo = mid + 1; else hi = mid;
  }
  for (int b = lo; b < B && p.cu[b] < s1; ++b) {
    const int sb = max(p.cu[b], 0);
    const int a = max(s0, sb), e = min(s1, p.cu[b + 1]);
    if (a >= e) continue;
    // ---- compact the valid positions of [a, e) (in order) into vpos, kSeg at a time
    if (tid == 0) hist_sh = history_before(p.mask, sb, a, W);
    int nvalid = 0;
    for (int a0 = a; a0 < e; a0 += kSeg) {
      const int pos = a0 + tid;
      const bool ok = pos < e && (p.mask == nullptr || p.mask[pos] != 0);
      const unsigned bits = __ballot_sync(0xFFFFFFFFu, ok);
      if (lane == 0) wcnt[warp] = __popc(bits);
      __syncthreads();
      int before = 0, tot = 0;
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) {
        before += (w < warp) ? wcnt[w] : 0;
        tot += wcnt[w];
      }
      if (ok) vpos[nvalid + before + __popc(bits & ((1u << lane) - 1u))] = pos;
      nvalid += tot;
      __syncthreads();     // wcnt is rewritten by the next pass
    }
    if (mine) {
      // ---- the window before the first valid row (oldest first)
      float win[kMaxW - 1][kPer];
#pragma unroll
      for (int j = 0; j < kMaxW - 1; ++j) {
#pragma unroll
        for (int q = 0; q < kPer; ++q) win[j][q] = 0.f;
        if (j < W - 1) {
          const int src = hist_sh.src[j];
          if (src >= 0) unpack_row<BF16>(load_row<BF16>(p.x, (size_t)src, D, c), win[j]);
          else if (p.state_in)
            unpack_row<false>(load_row<false>(p.state_in, (size_t)b * (W - 1) + (-1 - src), D, c), win[j]);
        }
      }
      // ---- walk the valid rows; ring[u] holds the raw load of row m0 + u
      constexpr int ring_n = BF16 ? kRing : kRing / 2;     // fp32 rows are twice as wide
      RawRow<BF16> ring[ring_n];
#pragma unroll
      for (int u = 0; u < ring_n; ++u)
        if (u < nvalid) ring[u] = load_row<BF16>(p.x, (size_t)vpos[u], D, c);
      for (int m0 = 0; m0 < nvalid; m0 += ring_n) {
#pragma unroll
        for (int u = 0; u < ring_n; ++u) {
          const int m = m0 + u;
          if (m < nvalid) {
            float xv[kPer], acc[kPer];
            unpack_row<BF16>(ring[u], xv);
            if (m + ring_n < nvalid) ring[u] = load_row<BF16>(p.x, (size_t)vpos[m + ring_n], D, c);
#pragma unroll
            for (int q = 0; q < kPer; ++q) acc[q] = fmaf(wx[q], xv[q], bz[q]);
            // taps: u_i = win[i] for i < W-1 (zero taps beyond), u_{W-1} = x_t
#pragma unroll
            for (int i = 0; i < kMaxW - 1; ++i)
#pragma unroll
              for (int q = 0; q < kPer; ++q) acc[q] = fmaf(wt[i][q], win[i][q], acc[q]);
            store_row<BF16>(p.y, (size_t)vpos[m], D, c, acc);
            // shift: the newest of the W-1 slots becomes x_t
#pragma unroll
            for (int j = 0; j < kMaxW - 2; ++j)
              if (j + 1 < W - 1) {
#pragma unroll
                for (int q = 0; q < kPer; ++q) win[j][q] = win[j + 1][q];
              }
#pragma unroll
            for (int j = 0; j < kMaxW - 1; ++j)
              if (j == W - 2) {
#pragma unroll
                for (int q = 0; q < kPer; ++q) win[j][q] = xv[q];
              }
          }
        }
      }
      // ---- pads: y = 0
      if (p.mask != nullptr && nvalid < e - a) {
        float z[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) z[q] = 0.f;
        for (int r = a; r < e; ++r)
          if (p.mask[r] == 0) store_row<BF16>(p.y, (size_t)r, D, c, z);
      }
    }
    __syncthreads();   // vpos, wcnt and hist_sh are rewritten by the next sequence
  }
}

// Kernel B: the new state, one thread per (sequence, channel); every old value a
// thread needs is read before it writes, so state_out may equal state_in.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) conv_state_kernel(ConvParams p) {
  const size_t idx = (size_t)blockIdx.x * kThreads + threadIdx.x;
  if (idx >= (size_t)p.num_seqs * p.D) return;
  const int b = (int)(idx / p.D), c = (int)(idx % p.D);
  const int W = p.W, need = W - 1;
  const int cb = p.cu[b], ce = p.cu[b + 1];
  if (b == 0 && c == 0 && p.cu[0] != 0) atomicOr(p.err, ERR_BIT_CHECK);
  if (cb > ce || cb < 0 || ce > p.N || (b == p.num_seqs - 1 && ce != p.N)) {
    if (c == 0) atomicOr(p.err, ERR_BIT_CHECK);
    return;
  }
  const Hist hs = history_before(p.mask, cb, ce, W);
  float v[kMaxW - 1];
#pragma unroll
  for (int j = 0; j < kMaxW - 1; ++j) {
    if (j >= need) break;
    const int src = hs.src[j];
    if (src >= 0) v[j] = load_elem<BF16>(p.x, (size_t)src * p.D + c);
    else v[j] = p.state_in ? p.state_in[((size_t)b * need + (-1 - src)) * p.D + c] : 0.f;
  }
#pragma unroll
  for (int j = 0; j < kMaxW - 1; ++j) {
    if (j >= need) break;
    p.state_out[((size_t)b * need + j) * p.D + c] = v[j];
  }
}

}  // namespace conv

cudaError_t launch_short_conv(const ConvParams &p, bool bf16, cudaStream_t s) {
  using namespace conv;
  if (p.N > 0) {
    // positions per CTA: about one wave of two CTAs per SM over the channel blocks,
    // at least 32 and at most kMaxSpan
    static int sms = 0;
    if (sms == 0) {
      int dev = 0, v = 0;
      if (cudaGetDevice(&dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        v = 148;
      sms = v;
    }
    const int cblocks = (p.D + kChan - 1) / kChan;
    const long long slots = (long long)2 * sms / cblocks > 0 ? (long long)2 * sms / cblocks : 1;
    long long span = ((long long)p.N + slots - 1) / slots;
    span = span < 32 ? 32 : (span > kMaxSpan ? kMaxSpan : span);
    const dim3 grid((unsigned)((p.N + span - 1) / span), (unsigned)cblocks);
    using Kern = void (*)(ConvParams, int);
    static const Kern kerns[2][4] = {
        {conv_kernel<false, 1>, conv_kernel<false, 2>, conv_kernel<false, 3>, conv_kernel<false, 4>},
        {conv_kernel<true, 1>, conv_kernel<true, 2>, conv_kernel<true, 3>, conv_kernel<true, 4>}};
    kerns[bf16 ? 1 : 0][p.W - 1]<<<grid, kThreads, 0, s>>>(p, (int)span);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.state_out && p.W > 1 && p.num_seqs > 0) {
    const size_t n = (size_t)p.num_seqs * p.D;
    const unsigned blocks = (unsigned)((n + kThreads - 1) / kThreads);
    if (bf16) conv_state_kernel<true><<<blocks, kThreads, 0, s>>>(p);
    else conv_state_kernel<false><<<blocks, kThreads, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace kda
