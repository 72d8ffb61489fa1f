// Backward pass of the KDA prefill: gradients of <o, dO> + <S_final, dS_final> with
// respect to q, k, v, log_alpha, beta and the initial state, by the blockwise
// (chunkwise) algorithm ("Kimi Linear wlasnie pokonal ...", remio.ai, section "Jak
// Kimi Linear wykorzystuje inteligentniejsza pamiec rekurencyjna": the same chunked
// form serves training).  Chunks of C = 64 rows; within a chunk, with g the
// cumulative log decay from the chunk start and P_ij = sum_c k_ic k_jc e^{g_ic - g_jc},
// Mf_ij = sum_c q_ic k_jc e^{g_ic - g_jc} (j <= i, every factor <= 1):
//   A = beta_i P_ij (j < i),  T = (I + A)^{-1},  T_b = T Diag(beta)
//   W = T_b (K e^g),  U_v = T_b V,  M = tril(Mf),  K~ = K e^{g_C - g},  gamma = e^{g_C}
//   U = U_v - W S,  O = (Q e^g) S + M U,  S' = Diag(gamma) S + K~^T U.
// Reverse mode of one chunk, with dS' the gradient of the state after it:
//   dU = M^T dO + K~ dS',  dS = (Q e^g)^T dO + Diag(gamma) dS' - W^T dU
//   d(Q e^g) = dO S^T,  dM = tril(dO U^T),  dK~ = U dS'^T,  dgamma = rowsum(S * dS')
//   dW = -dU S^T,  dT_b = dW (K e^g)^T + dU V^T,  d(K e^g) = T_b^T dW,  dV = T_b^T dU
//   dbeta_j = sum_i dT_b,ij T_ij + sum_{j'<j} dA_jj' P_jj',  dA = -T^T (dT_b Diag(beta)) T^T (j < i)
// and the pairwise terms of P and Mf, then the chain through e^{+-g} to q, k and g,
// and g to log_alpha by a reverse cumulative sum.
//
// Four kernels: (1) per (chunk, head), the chunk quantities W, Q e^g, K~, U_v, M, T,
// P, gamma (pairwise exponentials, so exact for any log_alpha <= 0); (2) per
// (sequence, head, 32 columns of d_v), the forward chain that stores the state at
// every chunk start; (3) the same CTAs walking the chunks backwards for dS' at every
// chunk end (and dS_0); (4) per (chunk, head), every gradient of the chunk's rows.
// Only (2) and (3) are serial over a sequence's chunks.  fp32 throughout; in (4) the
// dense products of each d_v slice run on the tensor cores in 3xTF32 (fp32 accuracy).
// Pads are identity steps (their inputs never read): zero gradients there.
#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace cbwd {

constexpr int C = 64;
constexpr int kThreads = 256;
constexpr int NS = 32;          // d_v columns per chain CTA
constexpr int LP = C + 1;       // padded length of a channel-major row

template <int DK, int DV>
struct Item {                   // per (chunk, head), fp32
  static constexpr size_t W = 0;                  // [C][DK]
  static constexpr size_t QG = W + C * DK;        // [C][DK]
  static constexpr size_t KT = QG + C * DK;       // [C][DK]
  static constexpr size_t UV = KT + C * DK;       // [C][DV]
  static constexpr size_t M = UV + C * DV;        // [C][C]
  static constexpr size_t T = M + C * C;          // [C][C]
  static constexpr size_t P = T + C * C;          // [C][C]
  static constexpr size_t GAM = P + C * C;        // [DK]
  static constexpr size_t FLOATS = GAM + DK;
};

// ---- workspace: chunk index | items | S at chunk starts | dS' at chunk ends
__host__ __device__ inline size_t max_chunks(int N, int B) { return (size_t)N / C + (size_t)B; }
__host__ __device__ inline size_t items_off(int B) { return ((size_t)(B + 1) * 4 + 255) / 256 * 256; }
__host__ __device__ inline size_t item_floats(int dk, int dv) {
  return (size_t)3 * C * dk + (size_t)C * dv + 3 * C * C + dk;
}
__host__ __device__ inline size_t states_off(int N, int B, int H, int dk, int dv) {
  return items_off(B) + max_chunks(N, B) * H * item_floats(dk, dv) * 4;
}
__host__ __device__ inline size_t dstates_off(int N, int B, int H, int dk, int dv) {
  return states_off(N, B, H, dk, dv) + max_chunks(N, B) * H * (size_t)dk * dv * 4;
}
__host__ __device__ inline size_t ws_total(int N, int B, int H, int dk, int dv) {
  return dstates_off(N, B, H, dk, dv) + max_chunks(N, B) * H * (size_t)dk * dv * 4;
}

// cbase[b] = chunks of sequences 0..b-1; checks cu_seqlens (non-decreasing, within N).
__global__ void __launch_bounds__(1024) index_kernel(BackwardParams p, int *cbase) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < p.num_seqs; b0 += 1024) {
    const int b = b0 + tid;
    int n = 0;
    if (b < p.num_seqs) {
      const int s = p.cu[b], e = p.cu[b + 1];
      if (s < 0 || e < s || e > p.N) atomicOr(p.err, ERR_BIT_CHECK);
      else n = (e - s + C - 1) / C;
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
      const int t = warp_tot[lane];
      int u = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, u, o);
        if (lane >= o) u += y;
      }
      warp_tot[lane] = u - t;
    }
    __syncthreads();
    const int excl = carry + warp_tot[w] + x - n;
    if (b < p.num_seqs) cbase[b] = excl;
    __syncthreads();
    if (tid == 1023) carry = excl + n;
    __syncthreads();
  }
  if (tid == 0) cbase[p.num_seqs] = carry;
}

// (global chunk index, head) of a per-chunk CTA -> sequence, first row, rows in the chunk.
struct ChunkPos {
  int b, r0, n;
};
__device__ __forceinline__ bool locate(const BackwardParams &p, const int *cbase, int gch, ChunkPos &cp) {
  if (gch >= cbase[p.num_seqs]) return false;
  int lo = 0, hi = p.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cbase[mid] <= gch) lo = mid; else hi = mid - 1;
  }
  cp.b = lo;
  cp.r0 = p.cu[lo] + (gch - cbase[lo]) * C;
  cp.n = min(C, p.cu[lo + 1] - cp.r0);
  return true;
}

__device__ __forceinline__ bool row_valid(const BackwardParams &p, const ChunkPos &cp, int r) {
  return r < cp.n && (p.mask == nullptr || p.mask[cp.r0 + r] != 0);
}

// Loads ROWS rows x W columns of a row-major array (bf16 or fp32) in 16-byte pieces, every
// piece of the thread in flight before the first is used, and hands each element to
// store(row, column, value); with MASKED, rows whose bit in vmask is clear read as 0.
// Element (r, c) is at first + r * stride + c.
template <bool BF16, int ROWS, int W, bool MASKED = true, typename F>
__device__ __forceinline__ void load_rows(const void *src, size_t first, size_t stride, uint64_t vmask,
                                          int tid, F store) {
  constexpr int V = BF16 ? 8 : 4, PER = W / V, TOTAL = ROWS * PER, K = (TOTAL + kThreads - 1) / kThreads;
  uint4 raw[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int e = tid + k * kThreads, r = e / PER, q = e % PER;
    raw[k] = make_uint4(0u, 0u, 0u, 0u);
    if (e < TOTAL && (!MASKED || ((vmask >> r) & 1ull)))
      raw[k] = __ldg(reinterpret_cast<const uint4 *>(static_cast<const char *>(src) +
                                                     (first + (size_t)r * stride + (size_t)q * V) * (BF16 ? 2 : 4)));
  }
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int e = tid + k * kThreads, r = e / PER, c0 = (e % PER) * V;
    if (e >= TOTAL) continue;
    const uint32_t w[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
    if constexpr (BF16) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        store(r, c0 + 2 * v, __uint_as_float(w[v] << 16));
        store(r, c0 + 2 * v + 1, __uint_as_float(w[v] & 0xFFFF0000u));
      }
    } else {
#pragma unroll
      for (int v = 0; v < 4; ++v) store(r, c0 + v, __uint_as_float(w[v]));
    }
  }
}

__device__ __forceinline__ uint64_t valid_rows(const BackwardParams &p, const ChunkPos &cp) {
  uint64_t m = 0;
  for (int r = 0; r < cp.n; ++r)
    if (p.mask == nullptr || p.mask[cp.r0 + r] != 0) m |= 1ull << r;
  return m;
}

// log_alpha of the chunk into gT ([DK][LP], channel-major), then summed over rows into g.
template <int DK>
__device__ void load_gates(const BackwardParams &p, const ChunkPos &cp, int h, uint64_t vmask, float *gT,
                           int tid) {
  if (p.gate_head) {
    for (int e = tid; e < C * DK; e += kThreads) {
      const int r = e % C, c = e / C;
      gT[c * LP + r] = ((vmask >> r) & 1ull) ? p.log_alpha[(size_t)(cp.r0 + r) * p.H + h] : 0.f;
    }
  } else {
    load_rows<false, C, DK>(p.log_alpha, ((size_t)cp.r0 * p.H + h) * DK, (size_t)p.H * DK, vmask, tid,
                            [&](int r, int c, float x) { gT[c * LP + r] = x; });
  }
  __syncthreads();
  if (tid < DK) {
    float acc = 0.f;
    for (int r = 0; r < C; ++r) {
      acc += gT[tid * LP + r];
      gT[tid * LP + r] = acc;
    }
  }
  __syncthreads();
}

// ============================================================ (1) chunk quantities
template <int DK, int DV, bool BF16>
__global__ void __launch_bounds__(kThreads, 1) intra_kernel(BackwardParams p, const int *cbase, float *items) {
  using IT = Item<DK, DV>;
  extern __shared__ __align__(16) float sm[];
  float *kT = sm, *qT = kT + DK * LP, *gT = qT + DK * LP;
  float *vv = gT + DK * LP;                  // [C][DV]
  float *Ps = vv + C * DV, *Ms = Ps + C * LP, *Ts = Ms + C * LP;   // [C][LP]
  float *bs = Ts + C * LP;                   // [C]
  if (device_error_latched(p.err)) return;
  const int H = p.H, h = blockIdx.x % H, tid = threadIdx.x;
  ChunkPos cp;
  if (!locate(p, cbase, blockIdx.x / H, cp)) return;
  float *it = items + (size_t)blockIdx.x * IT::FLOATS;

  const uint64_t vmask = valid_rows(p, cp);
  const size_t first = (size_t)cp.r0 * H + h;
  load_rows<BF16, C, DV>(p.v, first * DV, (size_t)H * DV, vmask, tid, [&](int r, int c, float x) { vv[r * DV + c] = x; });
  load_rows<BF16, C, DK>(p.k, first * DK, (size_t)H * DK, vmask, tid, [&](int r, int c, float x) { kT[c * LP + r] = x; });
  load_rows<BF16, C, DK>(p.q, first * DK, (size_t)H * DK, vmask, tid, [&](int r, int c, float x) { qT[c * LP + r] = x; });
  if (tid < C) bs[tid] = ((vmask >> tid) & 1ull) ? p.beta[(size_t)(cp.r0 + tid) * H + h] : 0.f;
  load_gates<DK>(p, cp, h, vmask, gT, tid);

  // ---- P_ij, Mf_ij (j <= i) by 16-row blocks.  Pairs inside a block: e^{g_i - g_j} per
  // channel.  Rows i after the block of j: with L the log decay at the block's last row,
  // e^{g_i - g_j} = e^{g_i - L} e^{L - g_j} (both <= 1), so P and Mf over those rows are
  // products of staged factor tiles (32 channels at a time, staged in the T tile).
  for (int pr = tid; pr < 4 * 136; pr += kThreads) {
    const int b = pr / 136, q = pr % 136;
    int ii = 0;
    while ((ii + 1) * (ii + 2) / 2 <= q) ++ii;
    const int i = 16 * b + ii, j = 16 * b + (q - ii * (ii + 1) / 2);
    float sp = 0.f, smf = 0.f;
    for (int c = 0; c < DK; ++c) {
      const float e = __expf(gT[c * LP + i] - gT[c * LP + j]) * kT[c * LP + j];
      sp = fmaf(kT[c * LP + i], e, sp);
      smf = fmaf(qT[c * LP + i], e, smf);
    }
    Ps[i * LP + j] = sp;
    Ms[i * LP + j] = smf;
  }
  {
    constexpr int CH = 32, SL = CH + 1;
    float *Fs = Ts, *Gs = Ts + 16 * SL, *Hs = Gs + 48 * SL;     // [16][SL], [48][SL], [48][SL]
    const int jl = tid & 15, ig = tid >> 4;
    for (int bs0 = 0; bs0 < 3; ++bs0) {
      const int j0 = 16 * bs0, i0 = j0 + 16, nr = C - i0, L = j0 + 15;
      float ap[3] = {0.f, 0.f, 0.f}, am[3] = {0.f, 0.f, 0.f};
      for (int c0 = 0; c0 < DK; c0 += CH) {
        __syncthreads();       // the previous chunk's tiles are read
        for (int e = tid; e < (16 + nr) * CH; e += kThreads) {
          const int r = e / CH, cc = e % CH, c = c0 + cc;
          const float gl = gT[c * LP + L];
          if (r < 16) {
            Fs[r * SL + cc] = kT[c * LP + j0 + r] * __expf(gl - gT[c * LP + j0 + r]);
          } else {
            const int i = i0 + r - 16;
            const float a = __expf(gT[c * LP + i] - gl);
            Gs[(r - 16) * SL + cc] = kT[c * LP + i] * a;
            Hs[(r - 16) * SL + cc] = qT[c * LP + i] * a;
          }
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          const int r = ig + 16 * m;
          if (r < nr) {
#pragma unroll 8
            for (int cc = 0; cc < CH; ++cc) {
              const float f = Fs[jl * SL + cc];
              ap[m] = fmaf(Gs[r * SL + cc], f, ap[m]);
              am[m] = fmaf(Hs[r * SL + cc], f, am[m]);
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 3; ++m) {
        const int r = ig + 16 * m;
        if (r < nr) {
          Ps[(i0 + r) * LP + j0 + jl] = ap[m];
          Ms[(i0 + r) * LP + j0 + jl] = am[m];
        }
      }
    }
  }
  __syncthreads();
  // ---- M and P out; Q e^g, K~, gamma out; K e^g row-major (in place of q) for the W product
  for (int e = tid; e < C * C; e += kThreads) {
    const int i = e / C, j = e % C;
    it[IT::M + e] = j <= i ? Ms[i * LP + j] : 0.f;
    it[IT::P + e] = j < i ? Ps[i * LP + j] : 0.f;
    Ts[i * LP + j] = 0.f;
  }
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, c = e % DK;
    const float g = gT[c * LP + r], gC = gT[c * LP + C - 1];
    it[IT::QG + e] = qT[c * LP + r] * __expf(g);
    it[IT::KT + e] = kT[c * LP + r] * __expf(gC - g);
  }
  if (tid < DK) it[IT::GAM + tid] = __expf(gT[tid * LP + C - 1]);
  __syncthreads();
  float *kg = qT;                              // [C][DK + 4], K e^g row-major
  constexpr int KGL = DK + 4;
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, c = e % DK;
    kg[r * KGL + c] = kT[c * LP + r] * __expf(gT[c * LP + r]);
  }
  // ---- T = (I + A)^{-1}, A_ij = beta_i P_ij (j < i), by doubling: 16 x 16 diagonal
  // blocks by forward substitution (a thread per column), then T21 = -T22 A21 T11 for the
  // 32 x 32 blocks and the 64 x 64 matrix (Ms is the scratch X = A21 T11)
  if (tid < C) {
    const int b0 = tid & ~15, j = tid;
    Ts[j * LP + j] = 1.f;
    for (int i = j + 1; i < b0 + 16; ++i) {
      float s = 0.f;
      for (int m = j; m < i; ++m) s = fmaf(Ps[i * LP + m], Ts[m * LP + j], s);
      Ts[i * LP + j] = -bs[i] * s;
    }
  }
  __syncthreads();
  for (int half = 16; half < C; half *= 2) {
    // blocks of 2*half: rows/cols [o, o + 2 half); X = A21 T11 (half x half), T21 = -T22 X
    const int nblk = C / (2 * half), outs = nblk * half * half;
    for (int e = tid; e < outs; e += kThreads) {
      const int bl = e / (half * half), r = (e / half) % half, cc = e % half;
      const int o = bl * 2 * half, i = o + half + r, j = o + cc;
      float s = 0.f;
      for (int m = cc; m < half; ++m) s = fmaf(Ps[i * LP + o + m], Ts[(o + m) * LP + j], s);
      Ms[i * LP + j] = bs[i] * s;
    }
    __syncthreads();
    for (int e = tid; e < outs; e += kThreads) {
      const int bl = e / (half * half), r = (e / half) % half, cc = e % half;
      const int o = bl * 2 * half, i = o + half + r, j = o + cc;
      float s = 0.f;
      for (int m = 0; m <= r; ++m) s = fmaf(Ts[i * LP + o + half + m], Ms[(o + half + m) * LP + j], s);
      Ts[i * LP + j] = -s;
    }
    __syncthreads();
  }
  for (int e = tid; e < C * C; e += kThreads) it[IT::T + e] = Ts[(e / C) * LP + e % C];
  // ---- W = T_b (K e^g), U_v = T_b V: thread (4 rows, 8 columns)
  {
    const int cb = tid & 15, i0 = (tid >> 4) * 4, c0 = cb * 8;
    auto product = [&](const float *src, int ld, int ncol, size_t off, int ldo) {
      if (c0 >= ncol) return;
      float acc[4][8];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[a][u] = 0.f;
      for (int j = 0; j <= i0 + 3; ++j) {
        const float4 x0 = *reinterpret_cast<const float4 *>(src + j * ld + c0);
        const float4 x1 = *reinterpret_cast<const float4 *>(src + j * ld + c0 + 4);
        const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        const float bj = bs[j];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const float t = Ts[(i0 + a) * LP + j] * bj;
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[a][u] = fmaf(t, xs[u], acc[a][u]);
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        float *dst = it + off + (size_t)(i0 + a) * ldo + c0;
        *reinterpret_cast<float4 *>(dst) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
      }
    };
    __syncthreads();
    product(kg, KGL, DK, IT::W, DK);
    product(vv, DV, DV, IT::UV, DV);
  }
}

// ============================================================ (2) forward chain
// One CTA per (sequence, head, 32 columns of d_v): S at every chunk start into the
// workspace; the next chunk's W, K~, U_v slice and gamma arrive by cp.async while the
// current one runs.  Each thread holds a 2 x 4 block of U and a 4 x 4 block of S's update.
// Forward chain buffers (two): W and K~ ([C][DK + 4]), the U_v slice ([C][NS + 4]), gamma.
// Backward chain: two buffers of Q e^g and W ([C][DK], read as float4 along d_k), the dO
// slice and gamma; one of K~ ([C][DK + 4]) and M ([C][C]).
template <int DK, int DV>
struct ChainSmem {
  static constexpr int LD = DK + 4;
  static constexpr int TILE = C * LD;
  static constexpr int SLP = NS + 4;
  static constexpr int BUF = 2 * TILE + C * SLP + DK;
  static constexpr int FLOATS = 2 * BUF + DK * SLP + C * SLP;
};
template <int DK, int DV>
struct DChainSmem {
  static constexpr int LD = DK + 4, LQ = DK;
  static constexpr int SLP = NS + 4;
  static constexpr int BUF = 2 * C * LQ + C * SLP + DK;
  static constexpr int ABUF = C * LD + C * C;
  static constexpr int FLOATS = 2 * BUF + ABUF + DK * SLP + C * SLP;
};

__device__ __forceinline__ void cp_rows(float *dst, int ld_dst, const float *src, int ld_src, int rows,
                                        int cols, int tid) {
  const int q = cols / 4;
  for (int e = tid; e < rows * q; e += kThreads) {
    const int r = e / q, c4 = (e % q) * 4;
    tc::cp_async16(tc::smem_u32(dst + r * ld_dst + c4), src + (size_t)r * ld_src + c4, 16);
  }
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
states_kernel(BackwardParams p, const int *cbase, const float *items, float *states) {
  using IT = Item<DK, DV>;
  using SMc = ChainSmem<DK, DV>;
  constexpr int LD = SMc::LD, SLP = SMc::SLP;
  extern __shared__ __align__(16) float sm[];
  float *buf[2] = {sm, sm + SMc::BUF};
  float *S = sm + 2 * SMc::BUF;               // [DK][SLP]
  float *U = S + DK * SLP;                    // [C][SLP]
  if (device_error_latched(p.err)) return;
  const int tiles = DV / NS, sl = blockIdx.x % tiles, bh = blockIdx.x / tiles;
  const int b = bh / p.H, h = bh % p.H, n0 = sl * NS, tid = threadIdx.x;
  const int nch = (p.cu[b + 1] - p.cu[b] + C - 1) / C, cb = cbase[b];
  const float *I0 = p.init_state ? p.init_state + (size_t)bh * DK * DV : nullptr;
  for (int e = tid; e < DK * NS; e += kThreads) {
    const int c = e / NS, n = e % NS;
    S[c * SLP + n] = I0 ? I0[(size_t)c * DV + n0 + n] : 0.f;
  }
  auto load = [&](int j, float *bf) {
    const float *it = items + ((size_t)(cb + j) * p.H + h) * IT::FLOATS;
    cp_rows(bf, LD, it + IT::W, DK, C, DK, tid);
    cp_rows(bf + SMc::TILE, LD, it + IT::KT, DK, C, DK, tid);
    cp_rows(bf + 2 * SMc::TILE, SLP, it + IT::UV + n0, DV, C, NS, tid);
    cp_rows(bf + 2 * SMc::TILE + C * SLP, DK, it + IT::GAM, DK, 1, DK, tid);
    tc::cp_async_commit();
  };
  if (nch > 0) load(0, buf[0]);
  const int n4 = (tid & 7) * 4, i2 = (tid >> 3) * 2, c4 = (tid >> 3) * 4;
  for (int j = 0; j < nch; ++j) {
    float *bf = buf[j & 1];
    tc::cp_async_wait_all();
    __syncthreads();
    if (j + 1 < nch) load(j + 1, buf[(j + 1) & 1]);
    const float *Wt = bf, *Kt = bf + SMc::TILE, *Uv = bf + 2 * SMc::TILE, *gam = Uv + C * SLP;
    float *Sg = states + ((size_t)(cb + j) * p.H + h) * DK * DV + n0;
    for (int e = tid; e < DK * NS / 4; e += kThreads) {
      const int c = e / (NS / 4), q = (e % (NS / 4)) * 4;
      *reinterpret_cast<float4 *>(Sg + (size_t)c * DV + q) = *reinterpret_cast<const float4 *>(S + c * SLP + q);
    }
    {   // U = U_v - W S: rows i2, i2 + 1, columns n4 .. n4 + 3
      float a0[4], a1[4];
      const float4 u0 = *reinterpret_cast<const float4 *>(Uv + i2 * SLP + n4);
      const float4 u1 = *reinterpret_cast<const float4 *>(Uv + (i2 + 1) * SLP + n4);
      a0[0] = u0.x; a0[1] = u0.y; a0[2] = u0.z; a0[3] = u0.w;
      a1[0] = u1.x; a1[1] = u1.y; a1[2] = u1.z; a1[3] = u1.w;
#pragma unroll 4
      for (int c = 0; c < DK; ++c) {
        const float w0 = Wt[i2 * LD + c], w1 = Wt[(i2 + 1) * LD + c];
        const float4 sv = *reinterpret_cast<const float4 *>(S + c * SLP + n4);
        a0[0] = fmaf(-w0, sv.x, a0[0]); a0[1] = fmaf(-w0, sv.y, a0[1]);
        a0[2] = fmaf(-w0, sv.z, a0[2]); a0[3] = fmaf(-w0, sv.w, a0[3]);
        a1[0] = fmaf(-w1, sv.x, a1[0]); a1[1] = fmaf(-w1, sv.y, a1[1]);
        a1[2] = fmaf(-w1, sv.z, a1[2]); a1[3] = fmaf(-w1, sv.w, a1[3]);
      }
      *reinterpret_cast<float4 *>(U + i2 * SLP + n4) = make_float4(a0[0], a0[1], a0[2], a0[3]);
      *reinterpret_cast<float4 *>(U + (i2 + 1) * SLP + n4) = make_float4(a1[0], a1[1], a1[2], a1[3]);
    }
    __syncthreads();
    if (c4 < DK) {   // S <- Diag(gamma) S + K~^T U: rows c4 .. c4 + 3, columns n4 .. n4 + 3
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float4 sv = *reinterpret_cast<const float4 *>(S + (c4 + a) * SLP + n4);
        const float g = gam[c4 + a];
        acc[a][0] = g * sv.x; acc[a][1] = g * sv.y; acc[a][2] = g * sv.z; acc[a][3] = g * sv.w;
      }
#pragma unroll 4
      for (int i = 0; i < C; ++i) {
        const float4 kt = *reinterpret_cast<const float4 *>(Kt + i * LD + c4);
        const float4 uv = *reinterpret_cast<const float4 *>(U + i * SLP + n4);
        const float ks[4] = {kt.x, kt.y, kt.z, kt.w}, us[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) acc[a][bb] = fmaf(ks[a], us[bb], acc[a][bb]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4 *>(S + (c4 + a) * SLP + n4) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    }
  }
  tc::cp_async_wait_all();
}

// ============================================================ (3) backward chain
// Chunks in reverse: dS' (gradient of the state after chunk j) into the workspace, then
//   dU = M^T dO + K~ dS',  dS <- (Q e^g)^T dO + Diag(gamma) dS' - W^T dU.
// Buffers: K~ and M (one slot, reloaded for chunk j-1 once dU of chunk j is done), and Q e^g,
// W, the dO slice (zero on pads) and gamma (two slots, one chunk ahead).
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
dstates_kernel(BackwardParams p, const int *cbase, const float *items, float *dstates) {
  using IT = Item<DK, DV>;
  using SMc = DChainSmem<DK, DV>;
  constexpr int LD = SMc::LD, LQ = SMc::LQ, SLP = SMc::SLP;
  extern __shared__ __align__(16) float sm[];
  float *buf[2] = {sm, sm + SMc::BUF};
  float *Kt = sm + 2 * SMc::BUF, *Mt = Kt + C * LD;     // [C][LD], [C][C]
  float *dS = Kt + SMc::ABUF;             // [DK][SLP]
  float *dU = dS + DK * SLP;              // [C][SLP]
  if (device_error_latched(p.err)) return;
  const int tiles = DV / NS, sl = blockIdx.x % tiles, bh = blockIdx.x / tiles;
  const int b = bh / p.H, h = bh % p.H, n0 = sl * NS, tid = threadIdx.x, H = p.H;
  const int cs = p.cu[b], nrow = p.cu[b + 1] - cs;
  const int nch = (nrow + C - 1) / C, cb = cbase[b];
  const float *F = p.d_final_state ? p.d_final_state + (size_t)bh * DK * DV : nullptr;
  for (int e = tid; e < DK * NS; e += kThreads) {
    const int c = e / NS, n = e % NS;
    dS[c * SLP + n] = F ? F[(size_t)c * DV + n0 + n] : 0.f;
  }
  auto load_b = [&](int j, float *bf) {
    const float *it = items + ((size_t)(cb + j) * H + h) * IT::FLOATS;
    cp_rows(bf, LQ, it + IT::QG, DK, C, DK, tid);
    cp_rows(bf + C * LQ, LQ, it + IT::W, DK, C, DK, tid);
    cp_rows(bf + 2 * C * LQ + C * SLP, DK, it + IT::GAM, DK, 1, DK, tid);
    float *dO = bf + 2 * C * LQ;
    for (int e = tid; e < C * NS / 4; e += kThreads) {
      const int r = e / (NS / 4), q = (e % (NS / 4)) * 4, row = j * C + r;
      const bool ok = row < nrow && (p.mask == nullptr || p.mask[cs + row] != 0);
      const float *src = p.d_o + ((size_t)(cs + (ok ? row : 0)) * H + h) * DV + n0 + q;
      tc::cp_async16(tc::smem_u32(dO + r * SLP + q), src, ok ? 16u : 0u);
    }
    tc::cp_async_commit();
  };
  auto load_a = [&](int j) {
    const float *it = items + ((size_t)(cb + j) * H + h) * IT::FLOATS;
    cp_rows(Kt, LD, it + IT::KT, DK, C, DK, tid);
    cp_rows(Mt, C, it + IT::M, C, C, C, tid);
    tc::cp_async_commit();
  };
  const int n4 = (tid & 7) * 4, i2 = (tid >> 3) * 2, c4 = (tid >> 3) * 4;
  if (nch > 0) {
    load_b(nch - 1, buf[(nch - 1) & 1]);
    load_a(nch - 1);
  }
  for (int j = nch - 1; j >= 0; --j) {
    float *bf = buf[j & 1];
    tc::cp_async_wait_all();
    __syncthreads();
    if (j > 0) load_b(j - 1, buf[(j - 1) & 1]);
    float *dSg = dstates + ((size_t)(cb + j) * H + h) * DK * DV + n0;
    for (int e = tid; e < DK * NS / 4; e += kThreads) {
      const int c = e / (NS / 4), q = (e % (NS / 4)) * 4;
      *reinterpret_cast<float4 *>(dSg + (size_t)c * DV + q) = *reinterpret_cast<const float4 *>(dS + c * SLP + q);
    }
    const float *Qg = bf, *Wt = bf + C * LQ, *dO = bf + 2 * C * LQ, *gam = dO + C * SLP;
    {   // dU = M^T dO + K~ dS': rows i2, i2 + 1, columns n4 .. n4 + 3
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      for (int r = i2; r < C; ++r) {
        const float m0 = Mt[r * C + i2], m1 = Mt[r * C + i2 + 1];
        const float4 d = *reinterpret_cast<const float4 *>(dO + r * SLP + n4);
        a0[0] = fmaf(m0, d.x, a0[0]); a0[1] = fmaf(m0, d.y, a0[1]); a0[2] = fmaf(m0, d.z, a0[2]); a0[3] = fmaf(m0, d.w, a0[3]);
        a1[0] = fmaf(m1, d.x, a1[0]); a1[1] = fmaf(m1, d.y, a1[1]); a1[2] = fmaf(m1, d.z, a1[2]); a1[3] = fmaf(m1, d.w, a1[3]);
      }
#pragma unroll 4
      for (int c = 0; c < DK; ++c) {
        const float k0 = Kt[i2 * LD + c], k1 = Kt[(i2 + 1) * LD + c];
        const float4 d = *reinterpret_cast<const float4 *>(dS + c * SLP + n4);
        a0[0] = fmaf(k0, d.x, a0[0]); a0[1] = fmaf(k0, d.y, a0[1]); a0[2] = fmaf(k0, d.z, a0[2]); a0[3] = fmaf(k0, d.w, a0[3]);
        a1[0] = fmaf(k1, d.x, a1[0]); a1[1] = fmaf(k1, d.y, a1[1]); a1[2] = fmaf(k1, d.z, a1[2]); a1[3] = fmaf(k1, d.w, a1[3]);
      }
      *reinterpret_cast<float4 *>(dU + i2 * SLP + n4) = make_float4(a0[0], a0[1], a0[2], a0[3]);
      *reinterpret_cast<float4 *>(dU + (i2 + 1) * SLP + n4) = make_float4(a1[0], a1[1], a1[2], a1[3]);
    }
    __syncthreads();
    if (j > 0) load_a(j - 1);
    if (c4 < DK) {   // dS <- (Q e^g)^T dO + Diag(gamma) dS' - W^T dU: rows c4 .. c4 + 3
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const float4 sv = *reinterpret_cast<const float4 *>(dS + (c4 + a) * SLP + n4);
        const float g = gam[c4 + a];
        acc[a][0] = g * sv.x; acc[a][1] = g * sv.y; acc[a][2] = g * sv.z; acc[a][3] = g * sv.w;
      }
#pragma unroll 2
      for (int i = 0; i < C; ++i) {
        const float4 q = *reinterpret_cast<const float4 *>(Qg + i * LQ + c4);
        const float4 w = *reinterpret_cast<const float4 *>(Wt + i * LQ + c4);
        const float4 d = *reinterpret_cast<const float4 *>(dO + i * SLP + n4);
        const float4 u = *reinterpret_cast<const float4 *>(dU + i * SLP + n4);
        const float qs[4] = {q.x, q.y, q.z, q.w}, ws[4] = {w.x, w.y, w.z, w.w};
        const float ds[4] = {d.x, d.y, d.z, d.w}, us[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int bb = 0; bb < 4; ++bb) acc[a][bb] = fmaf(qs[a], ds[bb], fmaf(-ws[a], us[bb], acc[a][bb]));
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4 *>(dS + (c4 + a) * SLP + n4) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    }
  }
  tc::cp_async_wait_all();
  __syncthreads();
  if (p.g_init_state) {
    float *O = p.g_init_state + (size_t)bh * DK * DV + n0;
    for (int e = tid; e < DK * NS; e += kThreads) O[(size_t)(e / NS) * DV + e % NS] = dS[(e / NS) * SLP + e % NS];
  }
}

// ============================================================ (4) gradients of a chunk
// Phase 1, d_v in 32-column slices: U, dU and dV of the slice, and its share of the
// d_v-contractions d(Q e^g) = dO S^T, dK~ = U dS'^T, dW = -dU S^T (4 x DK/16 blocks per
// thread, in registers), dM = dO U^T and dO-part of dT_b = dU V^T (4 x 4 blocks), dgamma.
// W, K~, M, T of the chunk stay in shared memory.  Phase 2 (shared memory reused): the
// chain through T, the pairwise terms with one thread per channel, log_alpha's sums.
// 3xTF32 tensor-core product (mma.sync m16n8k8, fp32 accumulate): each fp32 operand is
// split x = hi + lo with hi = tf32(x), lo = tf32(x - hi), and d += ah bh + ah bl + al bh
// (the dropped al bl is below 2^-21 of the product), so the sums keep fp32 accuracy.
// Fragment layout (g = lane / 4, t = lane % 4): A a0 = X[g][t], a1 = X[g+8][t],
// a2 = X[g][t+4], a3 = X[g+8][t+4]; B b0 = Y[t][g], b1 = Y[t+4][g]; C c0 = C[g][2t],
// c1 = C[g][2t+1], c2 = C[g+8][2t], c3 = C[g+8][2t+1].
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(x - __uint_as_float(hi)));
}
__device__ __forceinline__ void mma_tf32_acc(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ void mma3_tf32(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                          const uint32_t (&bh)[2], const uint32_t (&bl)[2]) {
  mma_tf32_acc(d, ah, bl);
  mma_tf32_acc(d, al, bh);
  mma_tf32_acc(d, ah, bh);
}
// B fragment (k0 + t, k0 + t + 4; n = n0 + g) of B[k][n] = X[n][k] (X row-major [.][ld]), split.
__device__ __forceinline__ void load_bt_split(const float *X, int ld, int n0, int k0, int g, int t,
                                              uint32_t (&h)[2], uint32_t (&l)[2]) {
  split_tf32(X[(n0 + g) * ld + k0 + t], h[0], l[0]);
  split_tf32(X[(n0 + g) * ld + k0 + t + 4], h[1], l[1]);
}
// B fragment of B[k][n] = X[k][n] (X row-major [.][ld]), split.
__device__ __forceinline__ void load_b_split(const float *X, int ld, int n0, int k0, int g, int t,
                                             uint32_t (&h)[2], uint32_t (&l)[2]) {
  split_tf32(X[(k0 + t) * ld + n0 + g], h[0], l[0]);
  split_tf32(X[(k0 + t + 4) * ld + n0 + g], h[1], l[1]);
}
// A fragment of A[r][k] = X[k][r] (X row-major [.][ld]), split; with LOWER, only entries of
// the lower triangle of X (k >= r) are taken, the rest count as 0.
template <bool LOWER>
__device__ __forceinline__ void load_at_split(const float *X, int ld, int r0, int k0, int g, int t,
                                              uint32_t (&h)[4], uint32_t (&l)[4]) {
  const int rr[4] = {r0 + g, r0 + g + 8, r0 + g, r0 + g + 8};
  const int kc[4] = {k0 + t, k0 + t, k0 + t + 4, k0 + t + 4};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float x = (!LOWER || kc[e] >= rr[e]) ? X[kc[e] * ld + rr[e]] : 0.f;
    split_tf32(x, h[e], l[e]);
  }
}
// A fragment rows r0, r0 + 8 and columns k0 + t, k0 + t + 4 of a row-major [.][ld] tile, split.
__device__ __forceinline__ void load_a_split(const float *X, int ld, int r0, int k0, int t, uint32_t (&h)[4],
                                             uint32_t (&l)[4]) {
  split_tf32(X[r0 * ld + k0 + t], h[0], l[0]);
  split_tf32(X[(r0 + 8) * ld + k0 + t], h[1], l[1]);
  split_tf32(X[r0 * ld + k0 + t + 4], h[2], l[2]);
  split_tf32(X[(r0 + 8) * ld + k0 + t + 4], h[3], l[3]);
}

template <int DK, int DV>
struct GradSmem {
  static constexpr int LD = DK + 4, SPI = NS + 4, SPC = DK + 4;
  // phase 1 (T at 0 throughout)
  static constexpr int T0 = 0;
  static constexpr int W1 = T0 + C * LP, K1 = W1 + C * LD, M1 = K1 + C * LD;
  static constexpr int SS = M1 + C * LP, SDS = SS + NS * SPC;      // [NS][DK + 4]
  static constexpr int SDO = SDS + NS * SPC, SU = SDO + C * SPI, SDU = SU + C * SPI, SV = SDU + C * SPI;
  static constexpr int END1 = SV + C * SPI;
  // phase 2
  static constexpr int DQG = T0 + C * LP, DKT = DQG + C * DK, DW = DKT + C * DK;
  static constexpr int DM = DW + C * DK, DTB = DM + C * LP, GT = DTB + C * LP;
  static constexpr int KB = GT + DK * LP, DGC = KB + C * (DK + 1), END2 = DGC + DK;
  static constexpr int DGAM = (END1 > END2 ? END1 : END2), DBETA = DGAM + DK;
  static constexpr int FLOATS = DBETA + C;
};

// Pairwise terms of one channel, split by 16-row blocks.  With dP (strictly lower) and
// dM (lower) of the chunk, per channel c the sums
//   S1_i = sum_{j<=i} dP_ij k_j e^{g_i - g_j},  S2_i = sum_{j<=i} dM_ij k_j e^{g_i - g_j},
//   S3_j = sum_{i>=j} (dP_ij k_i + dM_ij q_i) e^{g_i - g_j}
// give d k_i += S1_i + S3_i, d q_i += S2_i, d g_i += k_i S1_i + q_i S2_i - k_i S3_i.  For j in
// an earlier block than i, with R = g at the last row before i's block,
// e^{g_i - g_j} = e^{g_i - R} e^{R - g_j}, both factors <= 1: those sums become dense
// products with per-row factors (no overflow, one exponential per row and block).  Pairs
// inside a block take e^{g_i - g_j} directly.  Results are added to shared memory
// atomically (both threads of a channel add to some rows).
struct PairCtx {
  const float *gc;        // g of the channel, rows 0..63 (stride 1)
  const float *kb;        // k, [C][KP]
  int KP, c, DK;
  const float *dP, *dM;   // [C][LP]
  float *dk, *dq, *dg;    // [C][DK]
};

// i-side sums for rows of block B (> 0) from rows j < 16 B
template <int B>
__device__ __forceinline__ void pair_cross_i(const PairCtx &x, const float *qrow) {
  constexpr int NJ = 16 * B;
  const float R = x.gc[NJ - 1];
  float y[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) y[j] = x.kb[j * x.KP + x.c] * __expf(R - x.gc[j]);
#pragma unroll 2
  for (int ii = 0; ii < 16; ++ii) {
    const int i = NJ + ii;
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      s1 = fmaf(x.dP[i * LP + j], y[j], s1);
      s2 = fmaf(x.dM[i * LP + j], y[j], s2);
    }
    const float a = __expf(x.gc[i] - R);
    s1 *= a;
    s2 *= a;
    atomicAdd(x.dk + i * x.DK + x.c, s1);
    atomicAdd(x.dq + i * x.DK + x.c, s2);
    atomicAdd(x.dg + i * x.DK + x.c, fmaf(x.kb[i * x.KP + x.c], s1, qrow[ii] * s2));
  }
}

// j-side sums for rows j < 16 B from the rows of block B
template <int B>
__device__ __forceinline__ void pair_cross_j(const PairCtx &x, const float *qrow) {
  constexpr int NJ = 16 * B;
  const float R = x.gc[NJ - 1];
  float z[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) z[j] = 0.f;
#pragma unroll 2
  for (int ii = 0; ii < 16; ++ii) {
    const int i = NJ + ii;
    const float a = __expf(x.gc[i] - R);
    const float ka = x.kb[i * x.KP + x.c] * a, qa = qrow[ii] * a;
#pragma unroll
    for (int j = 0; j < NJ; ++j) z[j] = fmaf(x.dP[i * LP + j], ka, fmaf(x.dM[i * LP + j], qa, z[j]));
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const float s3 = z[j] * __expf(R - x.gc[j]);
    atomicAdd(x.dk + j * x.DK + x.c, s3);
    atomicAdd(x.dg + j * x.DK + x.c, -x.kb[j * x.KP + x.c] * s3);
  }
}

// pairs inside block B (j <= i, both in the block)
template <int B>
__device__ __forceinline__ void pair_block(const PairCtx &x, const float *qrow) {
  constexpr int O = 16 * B;
  float kk[16], gg[16], s3[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    kk[r] = x.kb[(O + r) * x.KP + x.c];
    gg[r] = x.gc[O + r];
    s3[r] = 0.f;
  }
#pragma unroll
  for (int ii = 0; ii < 16; ++ii) {
    const int i = O + ii;
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int jj = 0; jj <= ii; ++jj) {
      const int j = O + jj;
      const float e = __expf(gg[ii] - gg[jj]);
      const float dp = x.dP[i * LP + j], dm = x.dM[i * LP + j];
      s1 = fmaf(dp * kk[jj], e, s1);
      s2 = fmaf(dm * kk[jj], e, s2);
      s3[jj] = fmaf(fmaf(dp, kk[ii], dm * qrow[ii]), e, s3[jj]);
    }
    atomicAdd(x.dk + i * x.DK + x.c, s1);
    atomicAdd(x.dq + i * x.DK + x.c, s2);
    atomicAdd(x.dg + i * x.DK + x.c, fmaf(kk[ii], s1, qrow[ii] * s2));
  }
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) {
    atomicAdd(x.dk + (O + jj) * x.DK + x.c, s3[jj]);
    atomicAdd(x.dg + (O + jj) * x.DK + x.c, -kk[jj] * s3[jj]);
  }
}

template <int DK, int DV, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
grad_kernel(BackwardParams p, const int *cbase, const float *items, const float *states,
            const float *dstates) {
  using IT = Item<DK, DV>;
  using G = GradSmem<DK, DV>;
  constexpr int LD = G::LD, SPI = G::SPI, SPC = G::SPC, KP = DK + 1, CW = DK / 16;
  extern __shared__ __align__(16) float sm[];
  float *Ts = sm + G::T0;
  float *dgam = sm + G::DGAM, *dbeta = sm + G::DBETA;
  if (device_error_latched(p.err)) return;
  const int H = p.H, h = blockIdx.x % H, tid = threadIdx.x;
  const size_t gidx = blockIdx.x;
  ChunkPos cp;
  if (!locate(p, cbase, (int)(gidx / H), cp)) return;
  const float *it = items + gidx * IT::FLOATS;
  const float *Sg = states + gidx * DK * DV, *dSg = dstates + gidx * DK * DV;
  const uint64_t vmask = valid_rows(p, cp);
  auto valid = [&](int r) { return (vmask >> r) & 1ull; };
  const size_t first = (size_t)cp.r0 * H + h;
  auto betaf = [&](int r) -> float { return valid(r) ? p.beta[(size_t)(cp.r0 + r) * H + h] : 0.f; };

  // ---- phase 1
  float *Wt = sm + G::W1, *Kt = sm + G::K1, *Mt = sm + G::M1;
  float *sS = sm + G::SS, *sdS = sm + G::SDS, *sdO = sm + G::SDO, *sU = sm + G::SU;
  float *sdU = sm + G::SDU, *sV = sm + G::SV;
  cp_rows(Wt, LD, it + IT::W, DK, C, DK, tid);
  cp_rows(Kt, LD, it + IT::KT, DK, C, DK, tid);
  tc::cp_async_commit();
  for (int e = tid; e < C * C; e += kThreads) {
    Mt[(e / C) * LP + e % C] = it[IT::M + e];
    Ts[(e / C) * LP + e % C] = it[IT::T + e];
  }
  if (tid < DK) dgam[tid] = 0.f;
  // rows i0 .. i0 + 3 and channels c0 .. c0 + CW - 1: the thread's share of the d(K e^g) product
  // (phase 2); rows (tid & 15) * 4 .. and columns (tid >> 4) * 4 .. of dT_b there
  const int rb = tid >> 4, cbk = tid & 15, i0 = rb * 4, c0 = cbk * CW;
  const int mi0 = (tid & 15) * 4, mj0 = (tid >> 4) * 4;
  // tensor-core accumulators over the d_v slices: warp wq owns n-tiles wq NTW .. of dQg, dK~
  // and dW (columns of 8 channels) and n-tile wq of dM and dT_b (columns of 8 rows), all four
  // 16-row m-tiles
  constexpr int NTW = DK / 64;
  const int lane = tid & 31, wq = tid >> 5, fg = lane >> 2, ft4 = lane & 3;
  float fq[4][NTW][4], fk[4][NTW][4], fw[4][NTW][4], fm[4][4], ft[4][4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) fq[m][nt][e] = fk[m][nt][e] = fw[m][nt][e] = 0.f;
      fm[m][e] = ft[m][e] = 0.f;
    }
  }
  for (int n0 = 0; n0 < DV; n0 += NS) {
    __syncthreads();     // previous slice's readers are done
    load_rows<false, DK, NS, false>(Sg, n0, DV, 0, tid, [&](int c, int n, float x) { sS[n * SPC + c] = x; });
    load_rows<false, DK, NS, false>(dSg, n0, DV, 0, tid, [&](int c, int n, float x) { sdS[n * SPC + c] = x; });
    load_rows<false, C, NS>(p.d_o, first * DV + n0, (size_t)H * DV, vmask, tid,
                            [&](int r, int n, float x) { sdO[r * SPI + n] = x; });
    load_rows<BF16, C, NS>(p.v, first * DV + n0, (size_t)H * DV, vmask, tid,
                           [&](int r, int n, float x) { sV[r * SPI + n] = x; });
    tc::cp_async_wait_all();
    __syncthreads();
    // U = U_v - W S, dU = M^T dO + K~ dS' and then dV = T_b^T dU on the tensor cores (3xTF32):
    // 64 x NS each, warp wq the 16-row m-tile wq / 2 and the two 8-column n-tiles of half wq % 2
    {
      const int r0 = (wq >> 1) * 16, nb0 = (wq & 1) * 16;
      float fu[2][4], fd[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) fu[nb][e] = fd[nb][e] = 0.f;
#pragma unroll 4
      for (int k0 = 0; k0 < DK; k0 += 8) {
        uint32_t awh[4], awl[4], akh[4], akl[4];
        load_a_split(Wt, LD, r0 + fg, k0, ft4, awh, awl);
        load_a_split(Kt, LD, r0 + fg, k0, ft4, akh, akl);
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          uint32_t bh[2], bl[2];
          load_bt_split(sS, SPC, nb0 + nb * 8, k0, fg, ft4, bh, bl);
          mma3_tf32(fu[nb], awh, awl, bh, bl);
          load_bt_split(sdS, SPC, nb0 + nb * 8, k0, fg, ft4, bh, bl);
          mma3_tf32(fd[nb], akh, akl, bh, bl);
        }
      }
#pragma unroll 4
      for (int k0 = 0; k0 < C; k0 += 8) {
        uint32_t amh[4], aml[4];
        load_at_split<false>(Mt, LP, r0, k0, fg, ft4, amh, aml);   // M is stored lower-triangular
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          uint32_t bh[2], bl[2];
          load_b_split(sdO, SPI, nb0 + nb * 8, k0, fg, ft4, bh, bl);
          mma3_tf32(fd[nb], amh, aml, bh, bl);
        }
      }
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = r0 + fg + (e >> 1) * 8, cc = nb0 + nb * 8 + 2 * ft4 + (e & 1);
          sU[r * SPI + cc] = __ldg(it + IT::UV + (size_t)r * DV + n0 + cc) - fu[nb][e];
          sdU[r * SPI + cc] = fd[nb][e];
        }
      __syncthreads();
      float fv[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) fv[nb][e] = 0.f;
#pragma unroll 4
      for (int k0 = 0; k0 < C; k0 += 8) {
        uint32_t ath[4], atl[4];
        load_at_split<true>(Ts, LP, r0, k0, fg, ft4, ath, atl);      // T: lower triangle only
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          uint32_t bh[2], bl[2];
          load_b_split(sdU, SPI, nb0 + nb * 8, k0, fg, ft4, bh, bl);
          mma3_tf32(fv[nb], ath, atl, bh, bl);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int jr = r0 + fg + (e >> 1) * 8;
        if (jr < cp.n) {
          const float bj = betaf(jr);
          float *dst = p.gv + ((size_t)(cp.r0 + jr) * H + h) * DV + n0 + nb0 + 2 * ft4 + (e & 1);
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) dst[nb * 8] = fv[nb][e] * bj;
        }
      }
    }
    // d_k-side shares of this slice on the tensor cores (3xTF32, K = the slice's NS columns):
    //   dQg += dO S^T, dK~ += U dS'^T, dW -= dU S^T (B = the slice of S or dS', [NS][DK]),
    //   dM += dO U^T, dT_b += dU V^T (B = U or V read transposed)
#pragma unroll
    for (int kk = 0; kk < NS; kk += 8) {
      uint32_t bsh[NTW][2], bsl[NTW][2], bdh[NTW][2], bdl[NTW][2], buh[2], bul[2], bvh[2], bvl[2];
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) {
        const int n = (wq * NTW + nt) * 8 + fg;
        split_tf32(sS[(kk + ft4) * SPC + n], bsh[nt][0], bsl[nt][0]);
        split_tf32(sS[(kk + ft4 + 4) * SPC + n], bsh[nt][1], bsl[nt][1]);
        split_tf32(sdS[(kk + ft4) * SPC + n], bdh[nt][0], bdl[nt][0]);
        split_tf32(sdS[(kk + ft4 + 4) * SPC + n], bdh[nt][1], bdl[nt][1]);
      }
      {
        const int j = wq * 8 + fg;
        split_tf32(sU[j * SPI + kk + ft4], buh[0], bul[0]);
        split_tf32(sU[j * SPI + kk + ft4 + 4], buh[1], bul[1]);
        split_tf32(sV[j * SPI + kk + ft4], bvh[0], bvl[0]);
        split_tf32(sV[j * SPI + kk + ft4 + 4], bvh[1], bvl[1]);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        uint32_t aoh[4], aol[4], auh[4], aul[4], adh[4], adl[4];
        load_a_split(sdO, SPI, m * 16 + fg, kk, ft4, aoh, aol);
        load_a_split(sU, SPI, m * 16 + fg, kk, ft4, auh, aul);
        load_a_split(sdU, SPI, m * 16 + fg, kk, ft4, adh, adl);
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
          mma3_tf32(fq[m][nt], aoh, aol, bsh[nt], bsl[nt]);
          mma3_tf32(fk[m][nt], auh, aul, bdh[nt], bdl[nt]);
          mma3_tf32(fw[m][nt], adh, adl, bsh[nt], bsl[nt]);
        }
        mma3_tf32(fm[m], aoh, aol, buh, bul);
        mma3_tf32(ft[m], adh, adl, bvh, bvl);
      }
    }
    if (tid < DK) {
      float s = 0.f;
      for (int nn = 0; nn < NS; ++nn) s = fmaf(sS[nn * SPC + tid], sdS[nn * SPC + tid], s);
      dgam[tid] += s;
    }
  }
  __syncthreads();

  // ---- phase 2: accumulators to shared memory; g (channel-major), K e^g
  float *dQg = sm + G::DQG, *dKt = sm + G::DKT, *dW = sm + G::DW;
  float *dM = sm + G::DM, *dTb = sm + G::DTB, *gT = sm + G::GT, *kb = sm + G::KB, *dgC = sm + G::DGC;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int r = m * 16 + fg;
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt) {
      const int c = (wq * NTW + nt) * 8 + 2 * ft4;
      dQg[r * DK + c] = fq[m][nt][0];
      dQg[r * DK + c + 1] = fq[m][nt][1];
      dQg[(r + 8) * DK + c] = fq[m][nt][2];
      dQg[(r + 8) * DK + c + 1] = fq[m][nt][3];
      dKt[r * DK + c] = fk[m][nt][0];
      dKt[r * DK + c + 1] = fk[m][nt][1];
      dKt[(r + 8) * DK + c] = fk[m][nt][2];
      dKt[(r + 8) * DK + c + 1] = fk[m][nt][3];
      dW[r * DK + c] = -fw[m][nt][0];
      dW[r * DK + c + 1] = -fw[m][nt][1];
      dW[(r + 8) * DK + c] = -fw[m][nt][2];
      dW[(r + 8) * DK + c + 1] = -fw[m][nt][3];
    }
    const int j = wq * 8 + 2 * ft4;
    dM[r * LP + j] = (j <= r) ? fm[m][0] : 0.f;
    dM[r * LP + j + 1] = (j + 1 <= r) ? fm[m][1] : 0.f;
    dM[(r + 8) * LP + j] = (j <= r + 8) ? fm[m][2] : 0.f;
    dM[(r + 8) * LP + j + 1] = (j + 1 <= r + 8) ? fm[m][3] : 0.f;
    dTb[r * LP + j] = ft[m][0];
    dTb[r * LP + j + 1] = ft[m][1];
    dTb[(r + 8) * LP + j] = ft[m][2];
    dTb[(r + 8) * LP + j + 1] = ft[m][3];
  }
  load_rows<BF16, C, DK>(p.k, first * DK, (size_t)H * DK, vmask, tid, [&](int r, int c, float x) { kb[r * KP + c] = x; });
  load_gates<DK>(p, cp, h, vmask, gT, tid);
  {   // dT_b += dW (K e^g)^T: thread (column jr, rows ig + 4 a)
    const int jr = tid & 63, ig = tid >> 6;
    float acc[C / 4];
#pragma unroll
    for (int a = 0; a < C / 4; ++a) acc[a] = 0.f;
    for (int c = 0; c < DK; ++c) {
      const float kg = kb[jr * KP + c] * __expf(gT[c * LP + jr]);
#pragma unroll
      for (int a = 0; a < C / 4; ++a) acc[a] = fmaf(dW[(ig + 4 * a) * DK + c], kg, acc[a]);
    }
#pragma unroll
    for (int a = 0; a < C / 4; ++a) dTb[(ig + 4 * a) * LP + jr] += acc[a];
  }
  {   // d(K e^g) = T_b^T dW: thread (rows i0 .. as jr, channels c0 ..); written after a barrier
    float acc[4][CW];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int u = 0; u < CW; ++u) acc[a][u] = 0.f;
    for (int i = i0; i < C; ++i) {
      float tv[4], wv[CW];
#pragma unroll
      for (int a = 0; a < 4; ++a) tv[a] = Ts[i * LP + i0 + a];
#pragma unroll
      for (int u = 0; u < CW; u += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(dW + i * DK + c0 + u);
        wv[u] = x.x; wv[u + 1] = x.y; wv[u + 2] = x.z; wv[u + 3] = x.w;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int u = 0; u < CW; ++u) acc[a][u] = fmaf(tv[a], wv[u], acc[a][u]);
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float bj = betaf(i0 + a);
#pragma unroll
      for (int u = 0; u < CW; ++u) dW[(i0 + a) * DK + c0 + u] = acc[a][u] * bj;
    }
  }
  if (tid < C) {   // dbeta (T_b part): sum_i dT_b,ij T_ij
    const int jr = tid;
    float s = 0.f;
    for (int i = jr; i < C; ++i) s = fmaf(dTb[i * LP + jr], Ts[i * LP + jr], s);
    dbeta[jr] = s;
  }
  __syncthreads();
  for (int e = tid; e < C * C; e += kThreads) dTb[(e / C) * LP + e % C] *= betaf(e % C);   // dT
  __syncthreads();
  {   // X = dT T^T (4 x 4 blocks), then dA = -T^T X, strictly lower
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) acc[a][bb] = 0.f;
    for (int m = 0; m < C; ++m) {
      float dv[4], tv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        dv[a] = dTb[(mi0 + a) * LP + m];
        tv[a] = Ts[(mj0 + a) * LP + m];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acc[a][bb] = fmaf(dv[a], tv[bb], acc[a][bb]);
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) dTb[(mi0 + a) * LP + mj0 + bb] = acc[a][bb];
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) acc[a][bb] = 0.f;
    for (int m = 0; m < C; ++m) {
      float tv[4], xv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        tv[a] = Ts[m * LP + mi0 + a];
        xv[a] = dTb[m * LP + mj0 + a];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acc[a][bb] = fmaf(tv[a], xv[bb], acc[a][bb]);
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int bb = 0; bb < 4; ++bb)
        dTb[(mi0 + a) * LP + mj0 + bb] = (mj0 + bb < mi0 + a) ? -acc[a][bb] : 0.f;
    __syncthreads();
  }
  if (tid < C) {   // dbeta += sum_j dA_ij P_ij
    const int i = tid;
    float s = 0.f;
    for (int jr = 0; jr < i; ++jr) s = fmaf(dTb[i * LP + jr], __ldg(it + IT::P + (size_t)i * C + jr), s);
    dbeta[i] += s;
  }
  // dP = beta_i dA; dg_C = colsum(dK~ * K~) + dgamma * gamma
  __syncthreads();
  for (int e = tid; e < C * C; e += kThreads) dTb[(e / C) * LP + e % C] *= betaf(e / C);
  if (tid < DK) {
    const int c = tid;
    const float gC = gT[c * LP + C - 1];
    float s = dgam[c] * __expf(gC);
    for (int r = 0; r < C; ++r) s = fmaf(dKt[r * DK + c], kb[r * KP + c] * __expf(gC - gT[c * LP + r]), s);
    dgC[c] = s;
  }
  __syncthreads();
  // ---- the chain through e^{+-g} (elementwise, in place), then the pairwise terms (two
  // threads per channel, rows as i in [0, 45) and [45, 64) for the elementwise pass).
  const int c = tid % 128, half = tid / 128;
  const int ia = half ? 45 : 0, ib = half ? C : 45;
  if (c < DK) {
    const float gC = gT[c * LP + C - 1];
    for (int i = ia; i < ib; ++i) {
      const float gi = gT[c * LP + i], ki = kb[i * KP + c];
      const float qi = valid(i) ? load_elem<BF16>(p.q, (first + (size_t)i * H) * DK + c) : 0.f;
      const float eg = __expf(gi), et = __expf(gC - gi);
      const float tq = dQg[i * DK + c], tk = dW[i * DK + c], tt = dKt[i * DK + c];
      dQg[i * DK + c] = tq * eg;
      dW[i * DK + c] = fmaf(tk, eg, tt * et);
      dKt[i * DK + c] = fmaf(tq, qi * eg, ki * fmaf(tk, eg, -tt * et));
    }
  }
  __syncthreads();
  if (c < DK) {
    // the channel's g as a contiguous row, q of the rows this thread's blocks read
    const PairCtx x{gT + c * LP, kb, KP, c, DK, dTb, dM, dW, dQg, dKt};
    float qrow[2][16];
    auto load_q = [&](int blk, float *dst) {
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int i = 16 * blk + r;
        dst[r] = valid(i) ? load_elem<BF16>(p.q, (first + (size_t)i * H) * DK + c) : 0.f;
      }
    };
    if (half == 0) {         // blocks 0, 1 inside; rows of blocks 1, 2 from earlier blocks
      load_q(0, qrow[0]);
      load_q(1, qrow[1]);
      pair_block<0>(x, qrow[0]);
      pair_block<1>(x, qrow[1]);
      pair_cross_i<1>(x, qrow[1]);
      pair_cross_j<1>(x, qrow[1]);
      load_q(2, qrow[0]);
      pair_cross_i<2>(x, qrow[0]);
      pair_cross_j<2>(x, qrow[0]);
    } else {                 // blocks 2, 3 inside; rows of block 3 from earlier blocks
      load_q(2, qrow[0]);
      load_q(3, qrow[1]);
      pair_block<2>(x, qrow[0]);
      pair_block<3>(x, qrow[1]);
      pair_cross_i<3>(x, qrow[1]);
      pair_cross_j<3>(x, qrow[1]);
    }
  }
  __syncthreads();
  if (tid < DK) {   // g -> log_alpha: reverse cumulative sum, dg_C on every row
    float acc = dgC[tid];
    for (int r = C - 1; r >= 0; --r) {
      acc += dKt[r * DK + tid];
      dKt[r * DK + tid] = acc;
    }
  }
  __syncthreads();
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, cc = e % DK;
    if (r >= cp.n) continue;
    const bool ok = valid(r);
    const size_t row = (size_t)(cp.r0 + r) * H + h;
    p.gq[row * DK + cc] = ok ? dQg[r * DK + cc] : 0.f;
    p.gk[row * DK + cc] = ok ? dW[r * DK + cc] : 0.f;
    if (!p.gate_head) p.gla[row * DK + cc] = ok ? dKt[r * DK + cc] : 0.f;
  }
  if (tid < C && tid < cp.n) {
    const int r = tid;
    const bool ok = valid(r);
    const size_t row = (size_t)(cp.r0 + r) * H + h;
    p.gbeta[row] = ok ? dbeta[r] : 0.f;
    if (p.gate_head) {
      float s = 0.f;
      for (int cc = 0; cc < DK; ++cc) s += dKt[r * DK + cc];
      p.gla[row] = ok ? s : 0.f;
    }
  }
}

template <int DK, int DV, bool BF16>
cudaError_t launch(const BackwardParams &p, cudaStream_t s) {
  unsigned char *w = reinterpret_cast<unsigned char *>(p.ws);
  const int B = p.num_seqs;
  int *cbase = reinterpret_cast<int *>(w);
  float *items = reinterpret_cast<float *>(w + items_off(B));
  float *states = reinterpret_cast<float *>(w + states_off(p.N, B, p.H, DK, DV));
  float *dstates = reinterpret_cast<float *>(w + dstates_off(p.N, B, p.H, DK, DV));
  index_kernel<<<1, 1024, 0, s>>>(p, cbase);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t gch = max_chunks(p.N, B) * (size_t)p.H;
  if (gch > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  const int smem1 = (3 * DK * LP + C * DV + 3 * C * LP + C) * 4;
  if ((e = cudaFuncSetAttribute(intra_kernel<DK, DV, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem1)) != cudaSuccess)
    return e;
  intra_kernel<DK, DV, BF16><<<(unsigned)gch, kThreads, smem1, s>>>(p, cbase, items);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const unsigned gridc = (unsigned)B * p.H * (DV / NS);
  const int smem2 = ChainSmem<DK, DV>::FLOATS * 4, smem3 = DChainSmem<DK, DV>::FLOATS * 4;
  if ((e = cudaFuncSetAttribute(states_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2)) !=
      cudaSuccess)
    return e;
  states_kernel<DK, DV><<<gridc, kThreads, smem2, s>>>(p, cbase, items, states);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(dstates_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem3)) !=
      cudaSuccess)
    return e;
  dstates_kernel<DK, DV><<<gridc, kThreads, smem3, s>>>(p, cbase, items, dstates);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int smem4 = GradSmem<DK, DV>::FLOATS * 4;
  if ((e = cudaFuncSetAttribute(grad_kernel<DK, DV, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem4)) != cudaSuccess)
    return e;
  grad_kernel<DK, DV, BF16><<<(unsigned)gch, kThreads, smem4, s>>>(p, cbase, items, states, dstates);
  return cudaGetLastError();
}

}  // namespace cbwd

size_t backward_workspace(int N, int B, int H, int dk, int dv) { return cbwd::ws_total(N, B, H, dk, dv); }

cudaError_t launch_backward(const BackwardParams &p, bool bf16, cudaStream_t s) {
  using namespace cbwd;
  if (p.num_seqs == 0) return cudaSuccess;
#define KDA_BWD_CASE(DK_, DV_)                                                     \
  if (p.dk == DK_ && p.dv == DV_) return bf16 ? launch<DK_, DV_, true>(p, s) : launch<DK_, DV_, false>(p, s);
  KDA_BWD_CASE(64, 64)
  KDA_BWD_CASE(64, 128)
  KDA_BWD_CASE(128, 64)
  KDA_BWD_CASE(128, 128)
#undef KDA_BWD_CASE
  return cudaErrorNotSupported;
}

}  // namespace kda
