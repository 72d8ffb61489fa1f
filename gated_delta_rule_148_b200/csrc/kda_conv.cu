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
// kernel A gives each CTA 256 packed positions and up to 2048 channels; the pad
// mask of those positions is compacted once per CTA (warp ballots) into the list
// of valid rows, and each thread walks those rows for its 8 consecutive channels
// with the window in registers (one 16-byte load and one store per row).  Kernel B writes the new
// state after kernel A, one thread per (sequence, channel), so conv_state may be
// updated in place.
#include "kda_internal.cuh"

namespace kda {
namespace conv {

constexpr int kSeg = 256;            // packed positions per CTA
constexpr int kThreads = 256;
constexpr int kChan = 8 * kThreads;  // channels per CTA (8 per thread)
constexpr int kMaxW = 4;

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

template <bool BF16>
__device__ __forceinline__ void load8(const void *x, size_t row, int D, int c, float *v) {
  if (BF16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(x) + row * D + c));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = __uint_as_float(w[e] << 16);
      v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
  } else {
    const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + row * D + c);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <bool BF16>
__device__ __forceinline__ void store8(void *y, size_t row, int D, int c, const float *v) {
  if (BF16) {
    uint4 u;
    u.x = (uint32_t)f32_to_bf16_rne(v[0]) | ((uint32_t)f32_to_bf16_rne(v[1]) << 16);
    u.y = (uint32_t)f32_to_bf16_rne(v[2]) | ((uint32_t)f32_to_bf16_rne(v[3]) << 16);
    u.z = (uint32_t)f32_to_bf16_rne(v[4]) | ((uint32_t)f32_to_bf16_rne(v[5]) << 16);
    u.w = (uint32_t)f32_to_bf16_rne(v[6]) | ((uint32_t)f32_to_bf16_rne(v[7]) << 16);
    *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(y) + row * D + c) = u;
  } else {
    float4 *p = reinterpret_cast<float4 *>(reinterpret_cast<float *>(y) + row * D + c);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}


// Kernel A: outputs of packed positions [kSeg*blockIdx.x, +kSeg), channels
// [kChan*blockIdx.y, +kChan).  Thread t owns channels 8t .. 8t+7 and walks the
// CTA's valid rows in order with the window in registers, so each x row is read
// once; the 16-byte loads of one row are coalesced across the CTA's threads.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) conv_kernel(ConvParams p) {
  __shared__ int vpos[kSeg];
  __shared__ int wcnt[kThreads / 32];
  __shared__ Hist hist_sh;
  if (device_error_latched(p.err)) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int W = p.W, D = p.D, B = p.num_seqs;
  const int s0 = blockIdx.x * kSeg, s1 = min(s0 + kSeg, p.N);
  const int c_lo = blockIdx.y * kChan, nch = min(kChan, D - c_lo);
  if (blockIdx.x == 0 && blockIdx.y == 0) {       // cu_seqlens: 0, non-decreasing, ends at N
    bool bad = false;
    for (int b = tid; b < B; b += kThreads) bad |= p.cu[b] > p.cu[b + 1];
    if (tid == 0) bad |= p.cu[0] != 0 || p.cu[B] != p.N;
    if (bad) atomicOr(p.err, ERR_BIT_CHECK);
  }
  // this thread's channels and their taps
  const int cl = tid * 8, c = c_lo + cl;
  const bool mine = cl < nch;
  float wt[kMaxW - 1][8], wx[8], bz[8];      // window taps, the current row's tap, bias
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    bz[j] = (mine && p.bias) ? p.bias[c + j] : 0.f;
    wx[j] = mine ? p.weight[(size_t)(c + j) * W + (W - 1)] : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxW - 1; ++i) wt[i][j] = (mine && i < W - 1) ? p.weight[(size_t)(c + j) * W + i] : 0.f;
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
    // ---- compact the valid positions of [a, e) (in order) into vpos
    const int pos = a + tid;
    const bool ok = pos < e && (p.mask == nullptr || p.mask[pos] != 0);
    const unsigned bits = __ballot_sync(0xFFFFFFFFu, ok);
    if (lane == 0) wcnt[warp] = __popc(bits);
    if (tid == 0) hist_sh = history_before(p.mask, sb, a, W);
    __syncthreads();
    int before = 0, nvalid = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
      before += (w < warp) ? wcnt[w] : 0;
      nvalid += wcnt[w];
    }
    if (ok) vpos[before + __popc(bits & ((1u << lane) - 1u))] = pos;
    __syncthreads();
    if (mine) {
      // ---- the window before the first valid row (oldest first)
      float win[kMaxW - 1][8];
#pragma unroll
      for (int j = 0; j < kMaxW - 1; ++j) {
#pragma unroll
        for (int q = 0; q < 8; ++q) win[j][q] = 0.f;
        if (j < W - 1) {
          const int src = hist_sh.src[j];
          if (src >= 0) load8<BF16>(p.x, (size_t)src, D, c, win[j]);
          else if (p.state_in) load8<false>(p.state_in, (size_t)b * (W - 1) + (-1 - src), D, c, win[j]);
        }
      }
      // ---- walk the valid rows
#pragma unroll 2
      for (int m = 0; m < nvalid; ++m) {
        const size_t row = (size_t)vpos[m];
        float xv[8], acc[8];
        load8<BF16>(p.x, row, D, c, xv);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(wx[q], xv[q], bz[q]);
        // taps: u_i = win[i] for i < W-1 (zero taps beyond), u_{W-1} = x_t
#pragma unroll
        for (int i = 0; i < kMaxW - 1; ++i)
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[q] = fmaf(wt[i][q], win[i][q], acc[q]);
        store8<BF16>(p.y, row, D, c, acc);
        // shift: the newest of the W-1 slots becomes x_t
#pragma unroll
        for (int j = 0; j < kMaxW - 2; ++j)
          if (j + 1 < W - 1) {
#pragma unroll
            for (int q = 0; q < 8; ++q) win[j][q] = win[j + 1][q];
          }
#pragma unroll
        for (int j = 0; j < kMaxW - 1; ++j)
          if (j == W - 2) {
#pragma unroll
            for (int q = 0; q < 8; ++q) win[j][q] = xv[q];
          }
      }
      // ---- pads: y = 0
      if (p.mask != nullptr && nvalid < e - a) {
        const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int r = a; r < e; ++r)
          if (p.mask[r] == 0) store8<BF16>(p.y, (size_t)r, D, c, z);
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
    const dim3 grid((unsigned)((p.N + kSeg - 1) / kSeg), (unsigned)((p.D + kChan - 1) / kChan));
    if (bf16) conv_kernel<true><<<grid, kThreads, 0, s>>>(p);
    else conv_kernel<false><<<grid, kThreads, 0, s>>>(p);
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
