// KDA chunkwise prefill on the sm_100a tensor cores (tcgen05 / TMEM).
//
// The chunkwise WY/UT form ("Kimi Linear's 75% KV cache cut ...",
// theclarity.today, fourth paragraph: chunks plus the WY representation turn
// a chunk's rank-1 updates into a triangular solve and dense tensor-core
// products; "Kimi Linear wlasnie pokonal ...", remio.ai: blockwise algorithm
// with a diagonal-plus-low-rank transition).  Per chunk of C = 64 positions,
// incoming state S (d_k x d_v), g = inclusive per-channel cumsum of log_alpha
// inside the chunk, G = e^g, g_C = g at the chunk's last row:
//   A = beta * tril_{-1}((K G)(K e^{-g})^T),  M = tril_0((Q G)(K e^{-g})^T)
//   T_b = (I + A)^{-1} Diag(beta);  W = T_b (K G);  U_v = T_b V
//   U = U_v - W S;  O = (Q G) S + M U;  S <- Diag(e^{g_C}) S + (K e^{g_C - g})^T U
// One CTA (128 threads, one TMEM lane per thread) owns one (sequence, head,
// 64-column slice of d_v) and walks its chunks in order; S lives in TMEM as
// the fp32 accumulator of its own update for the whole sequence.
//
// Tensor-core products (M = 128 rows each, bf16 operands, fp32 accumulate):
//   Gram:  [Q G ; K G] (128 x 128) . (K e^{-g})^T          -> M (rows 0-63), A/beta (64-127)
//   W:     (K G)^T (128 x 64) . T_b^T                       -> W^T
//   U_v:   [T_b ; 0] (128 x 64) . V                         -> U_v (rows 0-63)
//   state: [-W ; Q G] (128 x 128) . S  (accumulated on U_v)  -> U (rows 0-63), (Q G) S (64-127)
//   out:   [0 ; M] (128 x 64) . U  (accumulated)            -> O (rows 64-127)
//   S:     (K e^{g_C-g})^T (128 x 64) . U  (accumulated on Diag(e^{g_C}) S)
// CUDA cores: the cumsum, the exponentials, masks, the 64 x 64 unit-lower
// inverse (fp32, blocked 16 x 16), bf16 packing and the epilogue.
//
// Exactness: masked and tail rows enter as zeros (and identity gates);
// upper-triangle entries are zeroed by selection before any product uses
// them, so an output row never depends on a later row's values.
// Numerical domain of this path: the factorisation e^{g_r - g_i} =
// e^{g_r} e^{-g_i} needs e^{-g} finite, i.e. a per-channel cumulative
// log-decay >= -80 within each 64-token chunk (the fp32 CUDA-core path has no
// such limit).
#include <climits>

#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kC = 64;       // chunk
constexpr int kDK = 128;     // key dim
constexpr int kNV = 64;      // d_v columns per CTA
constexpr int kThreads = 128;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 1.9 GHz

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_QKW = 0;                       // [-W | Q G | K G] 192 x 128 row tile
constexpr uint32_t OFF_KH = OFF_QKW + 192 * 256;      // K e^{-g}            64 x 128
constexpr uint32_t OFF_KT = OFF_KH + 64 * 256;        // K e^{g_C - g}       64 x 128
constexpr uint32_t OFF_TBM = OFF_KT + 64 * 256;       // [T_b | 0 | M]      192 x 64
constexpr uint32_t OFF_V = OFF_TBM + 192 * 128;       // V slice             64 x 64
constexpr uint32_t OFF_SB = OFF_V + 64 * 128;         // S (bf16)           128 x 64
constexpr uint32_t OFF_UB = OFF_SB + 128 * 128;       // U (bf16)            64 x 64
constexpr uint32_t OFF_STQ = OFF_UB + 64 * 128;       // staging q  [64][128] bf16
constexpr uint32_t OFF_STK = OFF_STQ + 64 * 256;      // staging k  [64][128] bf16
constexpr uint32_t OFF_STG = OFF_STK + 64 * 256;      // staging log_alpha -> g [64][128] f32
constexpr uint32_t OFF_STB = OFF_STG + 64 * 512;      // staging beta [64] f32
// The inverse scratch aliases the staging buffers: the next chunk is staged
// only after the inverse is done.
constexpr uint32_t OFF_AS = OFF_STQ;                  // A [64][65] f32 (in q/k staging)
constexpr uint32_t OFF_TS = OFF_STG;                  // T [64][65] f32 (in g staging)
constexpr uint32_t SMEM_USED = OFF_STB + 256;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;     // + alignment slack

// TMEM columns
constexpr uint32_t TM_S = 0, TM_D1 = 64, TM_G = 128, TM_W = 192, TM_COLS = 256;

__device__ __forceinline__ SeqSpan tc_span(const PrefillParams &p, int b) {
  if (p.spans) return p.spans[b];
  SeqSpan s;
  s.seq_begin = p.cu[b];
  s.begin = p.cu[b];
  s.end = p.cu[b + 1];
  s.pad_inside = 0;
  return s;
}

__device__ __forceinline__ bool row_valid(const PrefillParams &p, const SeqSpan &sp, int pos) {
  return pos < sp.end && (p.mask == nullptr || p.mask[pos] != 0);
}

// Stage q, k, log_alpha (and beta) of the chunk starting at c0 with cp.async;
// invalid rows are zero-filled without reading global memory.
__device__ __forceinline__ void stage_chunk(const PrefillParams &p, const SeqSpan &sp, int c0,
                                            int h, unsigned char *base, int tid) {
  const int H = p.H;
  const uint32_t sq = smem_u32(base + OFF_STQ), sk = smem_u32(base + OFF_STK);
  const uint32_t sg = smem_u32(base + OFF_STG);
  // q, k: 64 rows x 16 chunks of 16 B each
  for (int e = tid; e < kC * 16; e += kThreads) {
    const int r = e >> 4, ch = e & 15;
    const int pos = c0 + r;
    const bool ok = row_valid(p, sp, pos);
    const size_t gi = ((size_t)(ok ? pos : 0) * H + h) * kDK + ch * 8;
    cp_async16(sq + r * 256 + ch * 16, (const uint16_t *)p.q + gi, ok ? 16u : 0u);
    cp_async16(sk + r * 256 + ch * 16, (const uint16_t *)p.k + gi, ok ? 16u : 0u);
  }
  // log_alpha: 64 rows x 32 chunks of 16 B
  for (int e = tid; e < kC * 32; e += kThreads) {
    const int r = e >> 5, ch = e & 31;
    const int pos = c0 + r;
    const bool ok = row_valid(p, sp, pos);
    const size_t gi = ((size_t)(ok ? pos : 0) * H + h) * kDK + ch * 4;
    cp_async16(sg + r * 512 + ch * 16, p.log_alpha + gi, ok ? 16u : 0u);
  }
  if (tid < kC) {
    const int pos = c0 + tid;
    float* sb = reinterpret_cast<float *>(base + OFF_STB);
    sb[tid] = row_valid(p, sp, pos) ? p.beta[(size_t)pos * H + h] : 0.f;
  }
}

// V slice (64 rows x 64 columns) into the MN-major V tile.
__device__ __forceinline__ void stage_v(const PrefillParams &p, const SeqSpan &sp, int c0, int h,
                                        int dv0, unsigned char *base, int tid) {
  const uint32_t sv = smem_u32(base + OFF_V);
  for (int e = tid; e < kC * 8; e += kThreads) {
    const int r = e >> 3, ch = e & 7;
    const int pos = c0 + r;
    const bool ok = row_valid(p, sp, pos);
    const size_t gi = ((size_t)(ok ? pos : 0) * p.H + h) * p.dv + dv0 + ch * 8;
    cp_async16(sv + row_tile_chunk(r, 0, ch, kC), (const uint16_t *)p.v + gi, ok ? 16u : 0u);
  }
}

__device__ __forceinline__ void st_bf16(unsigned char *tile, uint32_t off, float x) {
  *reinterpret_cast<uint16_t *>(tile + off) = f32_to_bf16_rne(x);
}

// 64 x 64 unit-lower inverse T = (I + A)^{-1} in fp32, blocked by 16.
// A is strictly lower (row-major, stride 65) in As; T goes to Ts (stride 65).
__device__ void unit_lower_inverse(const float *As, float *Ts, int tid) {
  constexpr int S = 65;
  // diagonal 16 x 16 blocks: 64 threads, thread (blk, j) owns column j of block blk
  if (tid < 64) {
    const int blk = tid >> 4, j = tid & 15;
    const int o = blk * 16;
    for (int r = 0; r < 16; ++r) {
      float t;
      if (r < j) t = 0.f;
      else if (r == j) t = 1.f;
      else {
        t = 0.f;
        for (int i = j; i < r; ++i) t = fmaf(As[(o + r) * S + o + i], Ts[(o + i) * S + o + j], t);
        t = -t;
      }
      Ts[(o + r) * S + o + j] = t;
    }
  }
  __syncthreads();
  // off-diagonal blocks by distance d: T_ab = -D_a * sum_{m=b}^{a-1} A_am T_mb
  for (int d = 1; d <= 3; ++d) {
    const int nblk = 4 - d;                 // blocks (a, b) with a - b = d
    // X = sum_m A_am T_mb for each block: nblk * 256 entries; write into Ts block (a,b)
    // as a temporary, then multiply by D_a.
    __shared__ float X[3][16][17];
    for (int e = tid; e < nblk * 256; e += kThreads) {
      const int q = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      const int b = q, a = q + d;
      float acc = 0.f;
      for (int m = b; m < a; ++m)
        for (int i = 0; i < 16; ++i)
          acc = fmaf(As[(a * 16 + rr) * S + m * 16 + i], Ts[(m * 16 + i) * S + b * 16 + cc], acc);
      X[q][rr][cc] = acc;
    }
    __syncthreads();
    for (int e = tid; e < nblk * 256; e += kThreads) {
      const int q = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      const int b = q, a = q + d;
      float acc = 0.f;
      for (int i = 0; i <= rr; ++i) acc = fmaf(Ts[(a * 16 + rr) * S + a * 16 + i], X[q][i][cc], acc);
      Ts[(a * 16 + rr) * S + b * 16 + cc] = -acc;
    }
    __syncthreads();
  }
  // entries above the diagonal blocks are never read
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(PrefillParams p) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ float gC_sh[kDK];
  __shared__ float beta_sh[kC];

  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *base = smem_raw + pad;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;

  if (device_error_latched(p.err)) return;
  const int tiles = p.dv / kNV;
  const int tile = blockIdx.x % tiles;
  const int h = (blockIdx.x / tiles) % p.H;
  const int b = blockIdx.x / (tiles * p.H);
  const int dv0 = tile * kNV;
  const int H = p.H, DV = p.dv;
  const SeqSpan sp = tc_span(p, b);

  // ---- set-up: TMEM, barrier, zero rows of [T_b | 0 | M]
  if (warp == 0) tmem_alloc(&tmem_base_sh, TM_COLS);
  if (tid == 0) mbar_init(&mma_bar, 1);
  for (int e = tid; e < 64 * 8; e += kThreads) {     // rows 64..127 of TBM = 0
    const int r = 64 + (e >> 3), ch = e & 7;
    *reinterpret_cast<uint4 *>(base + OFF_TBM + row_tile_chunk(r, 0, ch, 192)) = make_uint4(0, 0, 0, 0);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = tmem_base_sh;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  uint32_t phase = 0;
  bool ok = true;

  // initial state into TMEM (thread tid owns state row tid)
  {
    float v[32];
    for (int half = 0; half < 2; ++half) {
      for (int j = 0; j < 32; ++j)
        v[j] = p.init_state ? p.init_state[(((size_t)b * H + h) * kDK + tid) * DV + dv0 + half * 32 + j]
                            : 0.f;
      tmem_st32(tm + lane_base + TM_S + half * 32, v);
    }
    tmem_st_wait();
  }

  const uint32_t sQKW = smem_u32(base + OFF_QKW), sKH = smem_u32(base + OFF_KH);
  const uint32_t sKT = smem_u32(base + OFF_KT), sTBM = smem_u32(base + OFF_TBM);
  const uint32_t sV = smem_u32(base + OFF_V), sSB = smem_u32(base + OFF_SB);
  const uint32_t sUB = smem_u32(base + OFF_UB);
  float *As = reinterpret_cast<float *>(base + OFF_AS);
  float *Ts = reinterpret_cast<float *>(base + OFF_TS);
  const float *stb = reinterpret_cast<const float *>(base + OFF_STB);
  static_assert(OFF_AS + 64 * 65 * 4 <= OFF_STG, "A scratch must fit the q/k staging");
  static_assert(OFF_TS + 64 * 65 * 4 <= OFF_STB, "T scratch must fit the g staging");

  if (sp.begin < sp.end) {
    stage_chunk(p, sp, sp.begin, h, base, tid);
    stage_v(p, sp, sp.begin, h, dv0, base, tid);
    cp_async_commit();
  }

  for (int c0 = sp.begin; c0 < sp.end; c0 += kC) {
    cp_async_wait_all();
    __syncthreads();
    // ---- P1: cumsum and operand tiles (thread = key channel)
    {
      const int c = tid;
      float *sg = reinterpret_cast<float *>(base + OFF_STG);
      float g = 0.f;
      for (int r = 0; r < kC; ++r) {
        g += sg[r * kDK + c];
        sg[r * kDK + c] = g;
      }
      const float gC = g;
      gC_sh[c] = gC;
      if (tid < kC) beta_sh[tid] = stb[tid];
      const uint16_t *sq = reinterpret_cast<const uint16_t *>(base + OFF_STQ);
      const uint16_t *sk = reinterpret_cast<const uint16_t *>(base + OFF_STK);
      for (int r = 0; r < kC; ++r) {
        const float gr = sg[r * kDK + c];
        const float qv = bf16_to_f32(sq[r * kDK + c]);
        const float kv = bf16_to_f32(sk[r * kDK + c]);
        const float e1 = __expf(gr);                   // <= 1
        const float e2 = __expf(gC - gr);              // <= 1
        const float e3 = __expf(fminf(-gr, 80.f));     // >= 1
        st_bf16(base + OFF_QKW, row_tile_off(64 + r, c, 192), qv * e1);
        st_bf16(base + OFF_QKW, row_tile_off(128 + r, c, 192), kv * e1);
        st_bf16(base + OFF_KH, row_tile_off(r, c, 64), kv * e3);
        st_bf16(base + OFF_KT, row_tile_off(r, c, 64), kv * e2);
      }
    }
    fence_async_smem();
    __syncthreads();
    // ---- Gram
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 64, 0, 0);
      for (int s = 0; s < 8; ++s)
        mma_bf16(tm + TM_G, desc_kmajor(sQKW, 192, 64, s), desc_kmajor(sKH, 64, 0, s), id, s > 0);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, kWaitCycles));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // ---- P3: M rows (lanes 0-63) -> TBM rows 128..191; A rows (lanes 64-127) -> As
    {
      float v[32];
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tm + lane_base + TM_G + half * 32, v);
        if (tid < kC) {
          const int r = tid;
          for (int j = 0; j < 32; j += 8) {
            uint4 pk;
            const int i0 = half * 32 + j;
            pk.x = pack_bf16x2(i0 + 0 <= r ? v[j + 0] : 0.f, i0 + 1 <= r ? v[j + 1] : 0.f);
            pk.y = pack_bf16x2(i0 + 2 <= r ? v[j + 2] : 0.f, i0 + 3 <= r ? v[j + 3] : 0.f);
            pk.z = pack_bf16x2(i0 + 4 <= r ? v[j + 4] : 0.f, i0 + 5 <= r ? v[j + 5] : 0.f);
            pk.w = pack_bf16x2(i0 + 6 <= r ? v[j + 6] : 0.f, i0 + 7 <= r ? v[j + 7] : 0.f);
            *reinterpret_cast<uint4 *>(base + OFF_TBM + row_tile_chunk(128 + r, 0, i0 >> 3, 192)) = pk;
          }
        } else {
          const int r = tid - kC;
          for (int j = 0; j < 32; ++j) {
            const int i = half * 32 + j;
            As[r * 65 + i] = (i < r) ? beta_sh[r] * v[j] : 0.f;
          }
        }
      }
    }
    __syncthreads();
    // ---- P4: T = (I + A)^{-1};  T_b = T Diag(beta) -> TBM rows 0..63
    unit_lower_inverse(As, Ts, tid);
    __syncthreads();
    {
      // thread pairs (row r, half): 64 rows x 2 halves of 32 columns
      const int r = tid >> 1, hh = tid & 1;
      for (int j = 0; j < 32; j += 8) {
        const int i0 = hh * 32 + j;
        float t[8];
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u;
          t[u] = (i <= r) ? Ts[r * 65 + i] * beta_sh[i] : 0.f;
        }
        uint4 pk;
        pk.x = pack_bf16x2(t[0], t[1]);
        pk.y = pack_bf16x2(t[2], t[3]);
        pk.z = pack_bf16x2(t[4], t[5]);
        pk.w = pack_bf16x2(t[6], t[7]);
        *reinterpret_cast<uint4 *>(base + OFF_TBM + row_tile_chunk(r, 0, i0 >> 3, 192)) = pk;
      }
    }
    fence_async_smem();
    __syncthreads();
    // the staging buffers are free: stream the next chunk's q, k, log_alpha, beta
    if (c0 + kC < sp.end) {
      stage_chunk(p, sp, c0 + kC, h, base, tid);
      cp_async_commit();
    }
    // ---- W^T = (K G)^T T_b^T ;  [U_v ; 0] = [T_b ; 0] V
    if (tid == 0) {
      fence_after_sync();
      const uint32_t idw = idesc_bf16(128, 64, 1, 0);
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + TM_W, desc_mnmajor(sQKW, 192, 128, s), desc_kmajor(sTBM, 192, 0, s), idw, s > 0);
      const uint32_t idu = idesc_bf16(128, 64, 0, 1);
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + TM_D1, desc_kmajor(sTBM, 192, 0, s), desc_mnmajor(sV, 64, 0, s), idu, s > 0);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, kWaitCycles));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // ---- P6: -W into QKW rows 0..63 (thread = channel c); S -> bf16 tile, S *= e^{g_C}
    {
      const int c = tid;
      float v[32];
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tm + lane_base + TM_W + half * 32, v);
        for (int j = 0; j < 32; ++j) st_bf16(base + OFF_QKW, row_tile_off(half * 32 + j, c, 192), -v[j]);
      }
      const float decay = __expf(gC_sh[c]);
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tm + lane_base + TM_S + half * 32, v);
        for (int j = 0; j < 32; j += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(v[j + 0], v[j + 1]);
          pk.y = pack_bf16x2(v[j + 2], v[j + 3]);
          pk.z = pack_bf16x2(v[j + 4], v[j + 5]);
          pk.w = pack_bf16x2(v[j + 6], v[j + 7]);
          *reinterpret_cast<uint4 *>(base + OFF_SB + row_tile_chunk(c, 0, (half * 32 + j) >> 3, 128)) = pk;
        }
        for (int j = 0; j < 32; ++j) v[j] *= decay;
        tmem_st32(tm + lane_base + TM_S + half * 32, v);
      }
      tmem_st_wait();
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    // V slice of the next chunk (the U_v product that read V is complete)
    if (c0 + kC < sp.end) {
      stage_v(p, sp, c0 + kC, h, dv0, base, tid);
      cp_async_commit();
    }
    // ---- [U ; (Q G) S] += [-W ; Q G] S
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 64, 0, 1);
      for (int s = 0; s < 8; ++s)
        mma_bf16(tm + TM_D1, desc_kmajor(sQKW, 192, 0, s), desc_mnmajor(sSB, 128, 0, s), id, 1);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, kWaitCycles));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // ---- P8: U (lanes 0-63) -> bf16 tile
    {
      float v[32];
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tm + lane_base + TM_D1 + half * 32, v);
        if (tid < kC) {
          for (int j = 0; j < 32; j += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(v[j + 0], v[j + 1]);
            pk.y = pack_bf16x2(v[j + 2], v[j + 3]);
            pk.z = pack_bf16x2(v[j + 4], v[j + 5]);
            pk.w = pack_bf16x2(v[j + 6], v[j + 7]);
            *reinterpret_cast<uint4 *>(base + OFF_UB + row_tile_chunk(tid, 0, (half * 32 + j) >> 3, 64)) = pk;
          }
        }
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    // ---- O += [0 ; M] U ;  S += (K e^{g_C - g})^T U
    if (tid == 0) {
      fence_after_sync();
      const uint32_t ido = idesc_bf16(128, 64, 0, 1);
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + TM_D1, desc_kmajor(sTBM, 192, 64, s), desc_mnmajor(sUB, 64, 0, s), ido, 1);
      const uint32_t ids = idesc_bf16(128, 64, 1, 1);
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + TM_S, desc_mnmajor(sKT, 64, 0, s), desc_mnmajor(sUB, 64, 0, s), ids, 1);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, kWaitCycles));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // ---- P10: O (lanes 64-127) -> global
    {
      float v[32];
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(tm + lane_base + TM_D1 + half * 32, v);
        if (tid >= kC) {
          const int r = tid - kC;
          const int pos = c0 + r;
          if (pos < sp.end) {
            const bool valid = p.mask == nullptr || p.mask[pos] != 0;
            uint16_t *orow = reinterpret_cast<uint16_t *>(p.o) + ((size_t)pos * H + h) * DV + dv0 + half * 32;
            for (int j = 0; j < 32; j += 8) {
              uint4 pk;
              pk.x = valid ? pack_bf16x2(v[j + 0], v[j + 1]) : 0u;
              pk.y = valid ? pack_bf16x2(v[j + 2], v[j + 3]) : 0u;
              pk.z = valid ? pack_bf16x2(v[j + 4], v[j + 5]) : 0u;
              pk.w = valid ? pack_bf16x2(v[j + 6], v[j + 7]) : 0u;
              *reinterpret_cast<uint4 *>(orow + j) = pk;
            }
          }
        }
      }
    }
    fence_before_sync();
    __syncthreads();
  }

  if (!ok) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_TIMEOUT);
    // let the product that timed out finish (bounded) before TMEM is released
    mbar_wait(&mma_bar, (phase - 1) & 1, kWaitCycles);
  } else if (p.final_state) {
    float v[32];
    for (int half = 0; half < 2; ++half) {
      tmem_ld32(tm + lane_base + TM_S + half * 32, v);
      float *dst = p.final_state + (((size_t)b * H + h) * kDK + tid) * DV + dv0 + half * 32;
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
  }
  cp_async_wait_all();
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, TM_COLS);
  }
}

}  // namespace

bool prefill_tc_supported(const PrefillParams &p, bool bf16) {
  return bf16 && p.dk == kDK && (p.dv % kNV) == 0 && p.chunk == kC;
}

cudaError_t launch_prefill_tc(const PrefillParams &p, cudaStream_t s) {
  if (p.num_seqs == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)p.num_seqs * p.H * (p.dv / kNV);
  prefill_tc_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
