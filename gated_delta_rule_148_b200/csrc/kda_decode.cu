// KDA single-token decode on a fixed-size fp32 state.
//
// One step per (row, head): S' = Diag(alpha) S; p = S'^T k;
// S = S' + k (beta (v - p))^T; o = S^T q  -- the per-channel decay, removal of
// the old projection onto the key and write of the new key-value pair of
// "Kimi Linear's 75% KV cache cut ..." (theclarity.today, third paragraph),
// on the fixed-size recurrent state of "Kimi Linear wlasnie pokonal pelna
// uwage ..." (remio.ai, the decode section).
//
// The step is HBM-bound: per active (row, head) the 64 KiB state (d = 128) is
// read once and written once; everything else is < 1 % of the bytes.  Design:
//   * one CTA of 256 threads per (row, head); the state tile never leaves
//     registers between its load and its store;
//   * thread t owns 4 consecutive dv columns (one 16-byte vector per state
//     row) and DK*DV/1024 rows, so every warp reads whole 512-byte rows
//     (DV = 128) -- fully coalesced, 16 independent 16-byte loads in flight
//     per thread before the first use;
//   * the two reductions over d_k (p = S'^T k and o = S^T q) are in-register
//     partial sums followed by one shared-memory pass across row groups;
//   * a masked row reads nothing from the state and writes only o = 0.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kDecodeThreads = 256;

template <int DK, int DV, bool BF16>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(DecodeParams p) {
  constexpr int TPR = DV / 4;                   // threads per state row (float4 each)
  constexpr int GROUPS = kDecodeThreads / TPR;  // row groups
  constexpr int RPT = DK / GROUPS;              // rows per thread
  static_assert(RPT * GROUPS == DK, "tiling");

  __shared__ float red[GROUPS][DV];
  __shared__ float s_k[DK], s_q[DK], s_a[DK];
  __shared__ float s_u[DV];

  const int bh = blockIdx.x;                // = b * H + h
  const int b = bh / p.H;
  const int tid = threadIdx.x;
  const int cg = tid % TPR;                 // column group: columns 4cg..4cg+3
  const int rg = tid / TPR;                 // row group: rows rg*RPT ...

  if (device_error_latched(p.err)) return;
  const bool active = (p.mask == nullptr) || (p.mask[b] != 0);
  if (!active) {
    for (int j = tid; j < DV; j += kDecodeThreads) store_elem<BF16>(p.o, (size_t)bh * DV + j, 0.f);
    return;
  }

  // state loads first: all RPT vectors in flight before any use
  float4 *S = reinterpret_cast<float4 *>(p.state + (size_t)bh * DK * DV);
  float4 s[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) s[i] = __ldcs(&S[(size_t)(rg * RPT + i) * TPR + cg]);

  for (int c = tid; c < DK; c += kDecodeThreads) {
    s_k[c] = load_elem<BF16>(p.k, (size_t)bh * DK + c);
    s_q[c] = load_elem<BF16>(p.q, (size_t)bh * DK + c);
    s_a[c] = __expf(p.log_alpha[p.gate_head ? (size_t)bh : (size_t)bh * DK + c]);
  }
  const float beta = p.beta[bh];
  __syncthreads();

  // decay and p = S'^T k (partial over this thread's rows)
  float pp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = rg * RPT + i;
    const float a = s_a[r], kr = s_k[r];
    s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
    pp[0] = fmaf(kr, s[i].x, pp[0]);
    pp[1] = fmaf(kr, s[i].y, pp[1]);
    pp[2] = fmaf(kr, s[i].z, pp[2]);
    pp[3] = fmaf(kr, s[i].w, pp[3]);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) red[rg][4 * cg + e] = pp[e];
  __syncthreads();
  for (int j = tid; j < DV; j += kDecodeThreads) {
    float acc = 0.f;
#pragma unroll
    for (int g = 0; g < GROUPS; ++g) acc += red[g][j];
    s_u[j] = beta * (load_elem<BF16>(p.v, (size_t)bh * DV + j) - acc);
  }
  __syncthreads();

  // rank-1 write, o partial, store
  float u[4] = {s_u[4 * cg], s_u[4 * cg + 1], s_u[4 * cg + 2], s_u[4 * cg + 3]};
  float oo[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = rg * RPT + i;
    const float kr = s_k[r], qr = s_q[r];
    s[i].x = fmaf(kr, u[0], s[i].x);
    s[i].y = fmaf(kr, u[1], s[i].y);
    s[i].z = fmaf(kr, u[2], s[i].z);
    s[i].w = fmaf(kr, u[3], s[i].w);
    oo[0] = fmaf(qr, s[i].x, oo[0]);
    oo[1] = fmaf(qr, s[i].y, oo[1]);
    oo[2] = fmaf(qr, s[i].z, oo[2]);
    oo[3] = fmaf(qr, s[i].w, oo[3]);
    __stcs(&S[(size_t)r * TPR + cg], s[i]);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) red[rg][4 * cg + e] = oo[e];
  __syncthreads();
  for (int j = tid; j < DV; j += kDecodeThreads) {
    float acc = 0.f;
#pragma unroll
    for (int g = 0; g < GROUPS; ++g) acc += red[g][j];
    store_elem<BF16>(p.o, (size_t)bh * DV + j, acc);
  }
}

template <int DK, int DV>
cudaError_t launch_dims(const DecodeParams &p, bool bf16, cudaStream_t s) {
  dim3 grid((unsigned)(p.B * p.H));
  if (bf16) decode_kernel<DK, DV, true><<<grid, kDecodeThreads, 0, s>>>(p);
  else decode_kernel<DK, DV, false><<<grid, kDecodeThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams &p, bool bf16, cudaStream_t s) {
  if (p.B == 0) return cudaSuccess;
  if (p.dk == 128 && p.dv == 128) return launch_dims<128, 128>(p, bf16, s);
  if (p.dk == 64 && p.dv == 64) return launch_dims<64, 64>(p, bf16, s);
  if (p.dk == 64 && p.dv == 128) return launch_dims<64, 128>(p, bf16, s);
  if (p.dk == 128 && p.dv == 64) return launch_dims<128, 64>(p, bf16, s);
  return cudaErrorInvalidValue;
}

}  // namespace kda
