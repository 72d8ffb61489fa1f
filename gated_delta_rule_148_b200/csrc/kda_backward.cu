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
// Only (2) and (3) are serial over a sequence's chunks.  fp32 on CUDA cores.
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

// Loads the chunk's k, q (channel-major, [DK][LP]) and log_alpha, summed into g; pads
// and rows past the sequence are identity steps (zeros).
template <int DK, bool BF16>
__device__ void load_keys(const BackwardParams &p, const ChunkPos &cp, int h, float *kT, float *qT,
                          float *gT, int tid) {
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, c = e % DK;
    float kv = 0.f, qv = 0.f, lv = 0.f;
    if (row_valid(p, cp, r)) {
      const size_t row = (size_t)(cp.r0 + r);
      kv = load_elem<BF16>(p.k, (row * p.H + h) * DK + c);
      qv = load_elem<BF16>(p.q, (row * p.H + h) * DK + c);
      lv = p.log_alpha[la_index(row, h, p.H, DK, c, p.gate_head)];
    }
    kT[c * LP + r] = kv;
    qT[c * LP + r] = qv;
    gT[c * LP + r] = lv;
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

  for (int e = tid; e < C * DV; e += kThreads) {
    const int r = e / DV, c = e % DV;
    vv[e] = row_valid(p, cp, r) ? load_elem<BF16>(p.v, ((size_t)(cp.r0 + r) * H + h) * DV + c) : 0.f;
  }
  if (tid < C) bs[tid] = row_valid(p, cp, tid) ? p.beta[(size_t)(cp.r0 + tid) * H + h] : 0.f;
  load_keys<DK, BF16>(p, cp, h, kT, qT, gT, tid);

  // ---- P_ij, Mf_ij (j <= i): rows rp and 63 - rp, columns j = jg + 8 m
  {
    const int rp = tid >> 3, jg = tid & 7;
    const int rows[2] = {rp, C - 1 - rp};
    float aP[2][8], aM[2][8];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int m = 0; m < 8; ++m) aP[a][m] = aM[a][m] = 0.f;
    for (int c = 0; c < DK; ++c) {
      const float *kc = kT + c * LP, *gc = gT + c * LP;
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int i = rows[a];
        const float gi = gc[i], ki = kc[i], qi = qT[c * LP + i];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int j = jg + 8 * m;
          if (j <= i) {
            const float e = __expf(gi - gc[j]) * kc[j];
            aP[a][m] = fmaf(ki, e, aP[a][m]);
            aM[a][m] = fmaf(qi, e, aM[a][m]);
          }
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int i = rows[a], j = jg + 8 * m;
        if (j <= i) {
          Ps[i * LP + j] = aP[a][m];
          Ms[i * LP + j] = aM[a][m];
        }
      }
  }
  __syncthreads();
  // ---- T = (I + A)^{-1}, A_ij = beta_i P_ij (j < i): column j by forward substitution
  if (tid < C) {
    const int j = tid;
    for (int i = 0; i < C; ++i) Ts[i * LP + j] = i == j ? 1.f : 0.f;
    for (int i = j + 1; i < C; ++i) {
      float s = 0.f;
      for (int m = j; m < i; ++m) s = fmaf(Ps[i * LP + m], Ts[m * LP + j], s);
      Ts[i * LP + j] = -bs[i] * s;
    }
  }
  __syncthreads();
  // ---- outputs that need no product: Q e^g, K~, gamma, M, T, P; then K e^g in place of k
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, c = e % DK;
    const float g = gT[c * LP + r], gC = gT[c * LP + C - 1];
    it[IT::QG + e] = qT[c * LP + r] * __expf(g);
    it[IT::KT + e] = kT[c * LP + r] * __expf(gC - g);
  }
  if (tid < DK) it[IT::GAM + tid] = __expf(gT[tid * LP + C - 1]);
  for (int e = tid; e < C * C; e += kThreads) {
    const int i = e / C, j = e % C;
    it[IT::M + e] = j <= i ? Ms[i * LP + j] : 0.f;
    it[IT::T + e] = Ts[i * LP + j];
    it[IT::P + e] = j < i ? Ps[i * LP + j] : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < C * DK; e += kThreads) {
    const int c = e / C, r = e % C;
    kT[c * LP + r] *= __expf(gT[c * LP + r]);
  }
  __syncthreads();
  // ---- W = T_b (K e^g), U_v = T_b V: thread (row half, column)
  {
    const int c = tid % 128, i0 = (tid / 128) * 32;
    if (c < DK) {
      for (int i = i0; i < i0 + 32; ++i) {
        float s = 0.f;
        for (int j = 0; j <= i; ++j) s = fmaf(Ts[i * LP + j] * bs[j], kT[c * LP + j], s);
        it[IT::W + (size_t)i * DK + c] = s;
      }
    }
    if (c < DV) {
      for (int i = i0; i < i0 + 32; ++i) {
        float s = 0.f;
        for (int j = 0; j <= i; ++j) s = fmaf(Ts[i * LP + j] * bs[j], vv[j * DV + c], s);
        it[IT::UV + (size_t)i * DV + c] = s;
      }
    }
  }
}

// ============================================================ (2) forward chain
// One CTA per (sequence, head, 32 columns of d_v): S at every chunk start into the
// workspace; the next chunk's W and K~ arrive by cp.async while the current one runs.
template <int DK, int DV>
struct ChainSmem {
  static constexpr int LD = DK + 4;                   // padded row of a [C][DK] tile
  static constexpr int TILE = C * LD;                 // floats
  static constexpr int BUF = 2 * TILE + C * NS + DK;  // W, K~ (or Q e^g, W), U_v / dO slice, gamma
  static constexpr int FLOATS = 2 * BUF + DK * NS + C * NS + C * LP;
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
  constexpr int LD = SMc::LD;
  extern __shared__ __align__(16) float sm[];
  float *buf[2] = {sm, sm + SMc::BUF};
  float *S = sm + 2 * SMc::BUF;           // [DK][NS]
  float *U = S + DK * NS;                 // [C][NS]
  if (device_error_latched(p.err)) return;
  const int tiles = DV / NS, sl = blockIdx.x % tiles, bh = blockIdx.x / tiles;
  const int b = bh / p.H, h = bh % p.H, n0 = sl * NS, tid = threadIdx.x;
  const int nch = (p.cu[b + 1] - p.cu[b] + C - 1) / C, cb = cbase[b];
  const float *I0 = p.init_state ? p.init_state + (size_t)bh * DK * DV : nullptr;
  for (int e = tid; e < DK * NS; e += kThreads) {
    const int c = e / NS, n = e % NS;
    S[e] = I0 ? I0[(size_t)c * DV + n0 + n] : 0.f;
  }
  auto load = [&](int j, float *bf) {
    const float *it = items + ((size_t)(cb + j) * p.H + h) * IT::FLOATS;
    cp_rows(bf, LD, it + IT::W, DK, C, DK, tid);
    cp_rows(bf + SMc::TILE, LD, it + IT::KT, DK, C, DK, tid);
    cp_rows(bf + 2 * SMc::TILE, NS, it + IT::UV + n0, DV, C, NS, tid);
    cp_rows(bf + 2 * SMc::TILE + C * NS, DK, it + IT::GAM, DK, 1, DK, tid);
    tc::cp_async_commit();
  };
  if (nch > 0) load(0, buf[0]);
  const int n = tid % NS, r0 = tid / NS;          // 8 row groups
  for (int j = 0; j < nch; ++j) {
    float *bf = buf[j & 1];
    tc::cp_async_wait_all();
    __syncthreads();
    if (j + 1 < nch) load(j + 1, buf[(j + 1) & 1]);
    const float *Wt = bf, *Kt = bf + SMc::TILE, *Uv = bf + 2 * SMc::TILE, *gam = Uv + C * NS;
    float *Sg = states + ((size_t)(cb + j) * p.H + h) * DK * DV + n0;
    for (int e = tid; e < DK * NS; e += kThreads) Sg[(size_t)(e / NS) * DV + e % NS] = S[e];
    // U = U_v - W S  (rows r0 + 8 m)
    for (int m = 0; m < C / 8; ++m) {
      const int i = r0 + 8 * m;
      float s = Uv[i * NS + n];
      for (int c = 0; c < DK; ++c) s = fmaf(-Wt[i * LD + c], S[c * NS + n], s);
      U[i * NS + n] = s;
    }
    __syncthreads();
    // S <- Diag(gamma) S + K~^T U  (rows r0 + 8 m of S)
    for (int m = 0; m < DK / 8; ++m) {
      const int c = r0 + 8 * m;
      float s = gam[c] * S[c * NS + n];
      for (int i = 0; i < C; ++i) s = fmaf(Kt[i * LD + c], U[i * NS + n], s);
      S[c * NS + n] = s;
    }
  }
  tc::cp_async_wait_all();
}

// ============================================================ (3) backward chain
// Chunks in reverse: dS' (gradient of the state after chunk j) into the workspace, then
//   dU = M^T dO + K~ dS',  dS <- (Q e^g)^T dO + Diag(gamma) dS' - W^T dU.
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
dstates_kernel(BackwardParams p, const int *cbase, const float *items, float *dstates) {
  using IT = Item<DK, DV>;
  using SMc = ChainSmem<DK, DV>;
  constexpr int LD = SMc::LD;
  extern __shared__ __align__(16) float sm[];
  float *buf[2] = {sm, sm + SMc::BUF};
  float *dS = sm + 2 * SMc::BUF;          // [DK][NS]
  float *dU = dS + DK * NS;               // [C][NS]
  float *Mt = dU + C * NS;                // [C][LP]
  if (device_error_latched(p.err)) return;
  const int tiles = DV / NS, sl = blockIdx.x % tiles, bh = blockIdx.x / tiles;
  const int b = bh / p.H, h = bh % p.H, n0 = sl * NS, tid = threadIdx.x, H = p.H;
  const int cs = p.cu[b], nrow = p.cu[b + 1] - cs;
  const int nch = (nrow + C - 1) / C, cb = cbase[b];
  const float *F = p.d_final_state ? p.d_final_state + (size_t)bh * DK * DV : nullptr;
  for (int e = tid; e < DK * NS; e += kThreads) {
    const int c = e / NS, n = e % NS;
    dS[e] = F ? F[(size_t)c * DV + n0 + n] : 0.f;
  }
  // buffer: Q e^g, W, dO slice, gamma; M separately (read after the buffer's tiles)
  auto load = [&](int j, float *bf) {
    const float *it = items + ((size_t)(cb + j) * H + h) * IT::FLOATS;
    cp_rows(bf, LD, it + IT::QG, DK, C, DK, tid);
    cp_rows(bf + SMc::TILE, LD, it + IT::W, DK, C, DK, tid);
    cp_rows(bf + 2 * SMc::TILE + C * NS, DK, it + IT::GAM, DK, 1, DK, tid);
    tc::cp_async_commit();
  };
  const int n = tid % NS, r0 = tid / NS;
  if (nch > 0) load(nch - 1, buf[(nch - 1) & 1]);
  for (int j = nch - 1; j >= 0; --j) {
    float *bf = buf[j & 1];
    const float *it = items + ((size_t)(cb + j) * H + h) * IT::FLOATS;
    // dO slice (pads and rows past the sequence are 0), M, K~ rows read from global below
    float *dO = bf + 2 * SMc::TILE;
    for (int e = tid; e < C * NS; e += kThreads) {
      const int r = e / NS, nn = e % NS, row = j * C + r;
      const bool ok = row < nrow && (p.mask == nullptr || p.mask[cs + row] != 0);
      dO[e] = ok ? p.d_o[((size_t)(cs + row) * H + h) * DV + n0 + nn] : 0.f;
    }
    for (int e = tid; e < C * C; e += kThreads) Mt[(e / C) * LP + e % C] = it[IT::M + e];
    tc::cp_async_wait_all();
    __syncthreads();
    if (j > 0) load(j - 1, buf[(j - 1) & 1]);
    float *dSg = dstates + ((size_t)(cb + j) * H + h) * DK * DV + n0;
    for (int e = tid; e < DK * NS; e += kThreads) dSg[(size_t)(e / NS) * DV + e % NS] = dS[e];
    const float *Qg = bf, *Wt = bf + SMc::TILE, *gam = dO + C * NS;
    const float *Kt = it + IT::KT;
    // dU = M^T dO + K~ dS'
    for (int m = 0; m < C / 8; ++m) {
      const int i = r0 + 8 * m;
      float s = 0.f;
      for (int r = i; r < C; ++r) s = fmaf(Mt[r * LP + i], dO[r * NS + n], s);
      const float *kr = Kt + (size_t)i * DK;
      for (int c = 0; c < DK; ++c) s = fmaf(__ldg(kr + c), dS[c * NS + n], s);
      dU[i * NS + n] = s;
    }
    __syncthreads();
    // dS <- (Q e^g)^T dO + Diag(gamma) dS' - W^T dU
    float nd[DK / 8];
#pragma unroll
    for (int m = 0; m < DK / 8; ++m) {
      const int c = r0 + 8 * m;
      float s = gam[c] * dS[c * NS + n];
      for (int i = 0; i < C; ++i) s = fmaf(Qg[i * LD + c], dO[i * NS + n], fmaf(-Wt[i * LD + c], dU[i * NS + n], s));
      nd[m] = s;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < DK / 8; ++m) dS[(r0 + 8 * m) * NS + n] = nd[m];
  }
  tc::cp_async_wait_all();
  __syncthreads();
  if (p.g_init_state) {
    float *O = p.g_init_state + (size_t)bh * DK * DV + n0;
    for (int e = tid; e < DK * NS; e += kThreads) O[(size_t)(e / NS) * DV + e % NS] = dS[e];
  }
}

// ============================================================ (4) gradients of a chunk
// Shared memory (fp32): the d_k-side accumulators dQg, dK~, dW ([C][DK]), dM, dT_b
// ([C][LP]), dgamma, dbeta; then d_v in 32-column slices: S, dS' ([DK][NS + 1]), dO, U,
// dU, V ([C][NS + 1]).  After the slices the slice region holds g (channel-major), T,
// K e^g (later k) ([C][DK + 1]) and dg_C.
constexpr int NSP = NS + 1;

template <int DK, int DV>
struct GradSmem {
  static constexpr int CT = C * DK;
  static constexpr int ACC = 3 * CT + 2 * C * LP + DK + C;
  static constexpr int SL = 2 * DK * NSP + 4 * C * NSP;
  static constexpr int PH2 = DK * LP + C * LP + C * (DK + 1) + DK;
  static constexpr int FLOATS = ACC + (SL > PH2 ? SL : PH2);
};

template <int DK, int DV, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
grad_kernel(BackwardParams p, const int *cbase, const float *items, const float *states,
            const float *dstates) {
  using IT = Item<DK, DV>;
  using G = GradSmem<DK, DV>;
  constexpr int KP = DK + 1;
  extern __shared__ __align__(16) float sm[];
  float *dQg = sm, *dKt = dQg + G::CT, *dW = dKt + G::CT;        // [C][DK]
  float *dM = dW + G::CT, *dTb = dM + C * LP;                     // [C][LP]
  float *dgam = dTb + C * LP, *dbeta = dgam + DK;                 // [DK], [C]
  float *reg = sm + G::ACC;
  float *sS = reg, *sdS = sS + DK * NSP;                          // [DK][NSP]
  float *sdO = sdS + DK * NSP, *sU = sdO + C * NSP, *sdU = sU + C * NSP, *sV = sdU + C * NSP;   // [C][NSP]
  float *gT = reg, *Ts = gT + DK * LP, *kb = Ts + C * LP, *dgC = kb + C * KP;
  if (device_error_latched(p.err)) return;
  const int H = p.H, h = blockIdx.x % H, tid = threadIdx.x;
  const size_t gidx = blockIdx.x;
  ChunkPos cp;
  if (!locate(p, cbase, (int)(gidx / H), cp)) return;
  const float *it = items + gidx * IT::FLOATS;
  const float *Sg = states + gidx * DK * DV, *dSg = dstates + gidx * DK * DV;
  uint64_t vmask = 0;       // valid rows of the chunk
  for (int r = 0; r < C; ++r)
    if (row_valid(p, cp, r)) vmask |= 1ull << r;
  auto valid = [&](int r) { return (vmask >> r) & 1ull; };
  auto betaf = [&](int r) -> float { return valid(r) ? p.beta[(size_t)(cp.r0 + r) * H + h] : 0.f; };

  for (int e = tid; e < G::ACC; e += kThreads) sm[e] = 0.f;
  __syncthreads();

  // ---- d_v slices: U, dU, dV and the slice's share of every d_v-contraction
  for (int n0 = 0; n0 < DV; n0 += NS) {
    for (int e = tid; e < DK * NS; e += kThreads) {
      const int c = e / NS, n = e % NS;
      sS[c * NSP + n] = Sg[(size_t)c * DV + n0 + n];
      sdS[c * NSP + n] = dSg[(size_t)c * DV + n0 + n];
    }
    for (int e = tid; e < C * NS; e += kThreads) {
      const int r = e / NS, n = e % NS;
      const bool ok = valid(r);
      const size_t row = (size_t)(cp.r0 + r) * H + h;
      sdO[r * NSP + n] = ok ? p.d_o[row * DV + n0 + n] : 0.f;
      sV[r * NSP + n] = ok ? load_elem<BF16>(p.v, row * DV + n0 + n) : 0.f;
    }
    __syncthreads();
    const int n = tid % NS, rg = tid / NS;
    for (int m = 0; m < C / 8; ++m) {            // U = U_v - W S
      const int i = rg + 8 * m;
      float s = it[IT::UV + (size_t)i * DV + n0 + n];
      const float *wr = it + IT::W + (size_t)i * DK;
      for (int c = 0; c < DK; ++c) s = fmaf(-__ldg(wr + c), sS[c * NSP + n], s);
      sU[i * NSP + n] = s;
    }
    for (int m = 0; m < C / 8; ++m) {            // dU = M^T dO + K~ dS'
      const int i = rg + 8 * m;
      float s = 0.f;
      for (int r = i; r < C; ++r) s = fmaf(__ldg(it + IT::M + (size_t)r * C + i), sdO[r * NSP + n], s);
      const float *kr = it + IT::KT + (size_t)i * DK;
      for (int c = 0; c < DK; ++c) s = fmaf(__ldg(kr + c), sdS[c * NSP + n], s);
      sdU[i * NSP + n] = s;
    }
    __syncthreads();
    for (int m = 0; m < C / 8; ++m) {            // dV = T_b^T dU
      const int jr = rg + 8 * m;
      if (jr >= cp.n) continue;
      float s = 0.f;
      for (int i = jr; i < C; ++i) s = fmaf(__ldg(it + IT::T + (size_t)i * C + jr), sdU[i * NSP + n], s);
      p.gv[((size_t)(cp.r0 + jr) * H + h) * DV + n0 + n] = s * betaf(jr);
    }
    {   // d_k-side shares: thread (row i, channel group cg)
      const int i = tid >> 2, cg = tid & 3;
      for (int c = cg; c < DK; c += 4) {
        float q = 0.f, kt = 0.f, w = 0.f;
#pragma unroll 8
        for (int nn = 0; nn < NS; ++nn) {
          const float sc = sS[c * NSP + nn];
          q = fmaf(sdO[i * NSP + nn], sc, q);
          kt = fmaf(sU[i * NSP + nn], sdS[c * NSP + nn], kt);
          w = fmaf(-sdU[i * NSP + nn], sc, w);
        }
        dQg[i * DK + c] += q;
        dKt[i * DK + c] += kt;
        dW[i * DK + c] += w;
      }
      for (int jr = cg; jr < C; jr += 4) {
        float mm = 0.f, tb = 0.f;
#pragma unroll 8
        for (int nn = 0; nn < NS; ++nn) {
          mm = fmaf(sdO[i * NSP + nn], sU[jr * NSP + nn], mm);
          tb = fmaf(sdU[i * NSP + nn], sV[jr * NSP + nn], tb);
        }
        if (jr <= i) dM[i * LP + jr] += mm;
        dTb[i * LP + jr] += tb;
      }
    }
    if (tid < DK) {
      float s = 0.f;
      for (int nn = 0; nn < NS; ++nn) s = fmaf(sS[tid * NSP + nn], sdS[tid * NSP + nn], s);
      dgam[tid] += s;
    }
    __syncthreads();
  }

  // ---- phase 2: g (channel-major), T, K e^g into the slice region
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, c = e % DK;
    gT[c * LP + r] = valid(r) ? p.log_alpha[la_index((size_t)(cp.r0 + r), h, H, DK, c, p.gate_head)] : 0.f;
  }
  for (int e = tid; e < C * C; e += kThreads) Ts[(e / C) * LP + e % C] = it[IT::T + e];
  __syncthreads();
  if (tid < DK) {
    float acc = 0.f;
    for (int r = 0; r < C; ++r) {
      acc += gT[tid * LP + r];
      gT[tid * LP + r] = acc;
    }
  }
  __syncthreads();
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, c = e % DK;
    kb[r * KP + c] = valid(r) ? load_elem<BF16>(p.k, ((size_t)(cp.r0 + r) * H + h) * DK + c) * __expf(gT[c * LP + r])
                              : 0.f;
  }
  __syncthreads();
  {   // dT_b += dW (K e^g)^T: thread (column jr, row group ig)
    const int jr = tid & 63, ig = tid >> 6;
    float acc[C / 4];
#pragma unroll
    for (int a = 0; a < C / 4; ++a) acc[a] = 0.f;
    for (int c = 0; c < DK; ++c) {
      const float kg = kb[jr * KP + c];
#pragma unroll
      for (int a = 0; a < C / 4; ++a) acc[a] = fmaf(dW[(ig + 4 * a) * DK + c], kg, acc[a]);
    }
#pragma unroll
    for (int a = 0; a < C / 4; ++a) dTb[(ig + 4 * a) * LP + jr] += acc[a];
  }
  __syncthreads();
  if (tid < DK) {   // d(K e^g) = T_b^T dW, in place of dW (thread per channel)
    const int c = tid;
    float col[C];
#pragma unroll
    for (int i = 0; i < C; ++i) col[i] = dW[i * DK + c];
#pragma unroll 4
    for (int jr = 0; jr < C; ++jr) {
      float s = 0.f;
      for (int i = jr; i < C; ++i) s = fmaf(Ts[i * LP + jr], col[i], s);
      dW[jr * DK + c] = s * betaf(jr);
    }
  } else if (tid - DK < C) {   // dbeta (T_b part): sum_i dT_b,ij T_ij
    const int jr = tid - DK;
    float s = 0.f;
    for (int i = jr; i < C; ++i) s = fmaf(dTb[i * LP + jr], Ts[i * LP + jr], s);
    dbeta[jr] = s;
  }
  __syncthreads();
  for (int e = tid; e < C * C; e += kThreads) dTb[(e / C) * LP + e % C] *= betaf(e % C);   // dT
  __syncthreads();
  if (tid < C) {   // X = dT T^T, in place (thread per row)
    const int i = tid;
    float row[C];
#pragma unroll
    for (int m = 0; m < C; ++m) row[m] = dTb[i * LP + m];
#pragma unroll 4
    for (int jr = 0; jr < C; ++jr) {
      float s = 0.f;
      for (int m = 0; m <= jr; ++m) s = fmaf(row[m], Ts[jr * LP + m], s);
      dTb[i * LP + jr] = s;
    }
  }
  __syncthreads();
  if (tid < C) {   // dA_ij = -sum_{m >= i} T_mi X_mj (j < i), in place (thread per column)
    const int jr = tid;
    float col[C];
#pragma unroll
    for (int m = 0; m < C; ++m) col[m] = dTb[m * LP + jr];
#pragma unroll 4
    for (int i = 0; i < C; ++i) {
      float s = 0.f;
      if (jr < i)
        for (int m = i; m < C; ++m) s = fmaf(Ts[m * LP + i], col[m], s);
      dTb[i * LP + jr] = -s;
    }
  }
  __syncthreads();
  if (tid < C) {   // dbeta += sum_j dA_ij P_ij
    const int i = tid;
    float s = 0.f;
    for (int jr = 0; jr < i; ++jr) s = fmaf(dTb[i * LP + jr], __ldg(it + IT::P + (size_t)i * C + jr), s);
    dbeta[i] += s;
  }
  // raw k replaces K e^g; dg_C = colsum(dK~ * K~) + dgamma * gamma
  for (int e = tid; e < C * DK; e += kThreads) {
    const int r = e / DK, c = e % DK;
    kb[r * KP + c] = valid(r) ? load_elem<BF16>(p.k, ((size_t)(cp.r0 + r) * H + h) * DK + c) : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < C * C; e += kThreads) dTb[(e / C) * LP + e % C] *= betaf(e / C);        // dP
  if (tid < DK) {
    const int c = tid;
    const float gC = gT[c * LP + C - 1];
    float s = dgam[c] * __expf(gC);
    for (int r = 0; r < C; ++r) s = fmaf(dKt[r * DK + c], kb[r * KP + c] * __expf(gC - gT[c * LP + r]), s);
    dgC[c] = s;
  }
  __syncthreads();
  auto qval = [&](int r, int c) -> float {
    return valid(r) ? load_elem<BF16>(p.q, ((size_t)(cp.r0 + r) * H + h) * DK + c) : 0.f;
  };
  // ---- pairwise terms with the chain through e^{+-g}; two threads per channel split the rows
  // (pairs j <= i: rows 0-44 and 45-63 as i, then rows 0-18 and 19-63 as j)
  const int c = tid % 128, half = tid / 128;
  if (c < DK) {
    const float gC = gT[c * LP + C - 1];
    const int ia = half ? 45 : 0, ib = half ? C : 45;
    for (int i = ia; i < ib; ++i) {
      const float gi = gT[c * LP + i], ki = kb[i * KP + c], qi = qval(i, c);
      float dk = 0.f, dq = 0.f, dg = 0.f;
      for (int jr = 0; jr <= i; ++jr) {
        const float e = __expf(gi - gT[c * LP + jr]) * kb[jr * KP + c];
        const float dp = dTb[i * LP + jr], dm = dM[i * LP + jr];    // dP is 0 on the diagonal
        dk = fmaf(dp, e, dk);
        dq = fmaf(dm, e, dq);
        dg = fmaf(fmaf(dp, ki, dm * qi), e, dg);
      }
      const float eg = __expf(gi), et = __expf(gC - gi);
      dq = fmaf(dQg[i * DK + c], eg, dq);
      dg = fmaf(dQg[i * DK + c], qi * eg, dg);
      dk = fmaf(dW[i * DK + c], eg, dk);
      dg = fmaf(dW[i * DK + c], ki * eg, dg);
      dk = fmaf(dKt[i * DK + c], et, dk);
      dg = fmaf(-dKt[i * DK + c], ki * et, dg);
      dQg[i * DK + c] = dq;
      dW[i * DK + c] = dk;
      dKt[i * DK + c] = dg;
    }
  }
  __syncthreads();
  if (c < DK) {
    const int ja = half ? 19 : 0, jb = half ? C : 19;
    for (int jr = ja; jr < jb; ++jr) {
      const float gj = gT[c * LP + jr], kj = kb[jr * KP + c];
      float dk = 0.f, dg = 0.f;
      for (int i = jr; i < C; ++i) {
        const float e = __expf(gT[c * LP + i] - gj);
        const float a = fmaf(dTb[i * LP + jr], kb[i * KP + c], dM[i * LP + jr] * qval(i, c));
        dk = fmaf(a, e, dk);
        dg = fmaf(a * kj, e, dg);
      }
      dW[jr * DK + c] += dk;
      dKt[jr * DK + c] -= dg;
    }
  }
  __syncthreads();
  // ---- g -> log_alpha (reverse cumulative sum, dg_C on every row), outputs
  if (tid < DK) {
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
  const int smem2 = ChainSmem<DK, DV>::FLOATS * 4;
  if ((e = cudaFuncSetAttribute(states_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2)) !=
      cudaSuccess)
    return e;
  states_kernel<DK, DV><<<gridc, kThreads, smem2, s>>>(p, cbase, items, states);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(dstates_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2)) !=
      cudaSuccess)
    return e;
  dstates_kernel<DK, DV><<<gridc, kThreads, smem2, s>>>(p, cbase, items, dstates);
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
