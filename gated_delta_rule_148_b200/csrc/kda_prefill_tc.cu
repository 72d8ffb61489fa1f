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
// CUDA cores: the cumsum, the exponentials, masks, bf16 packing and the
// epilogue; the 64 x 64 unit-lower inverse is blocked 16 x 16 with its block
// products on warp-level tensor-core MMAs (kda_tril_inv.cuh).
// 256 threads: thread t owns TMEM lane t % 128 and half (t / 128) of the
// 64 columns of every accumulator it reads.
//
// Exactness: masked and tail rows enter as zeros (and identity gates);
// upper-triangle entries are zeroed by selection before any product uses
// them, so an output row never depends on a later row's values.
// Range: the factorisation e^{g_r - g_i} = e^{g_r} e^{-g_i} is used for the
// channels whose log-decay over the chunk stays above about -60; the Gram terms
// of any other channel are computed exactly on the CUDA cores
// (prep::exact_gram_fixup), so the path holds for every log_alpha <= 0.
#include <climits>

#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "kda_tc.cuh"
#include "kda_tril_inv.cuh"
#include "kda_chunk_prep.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kC = 64;       // chunk
constexpr int kDK = 128;     // key dim
constexpr int kNV = 64;      // d_v columns per CTA
constexpr int kThreads = 256;

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
constexpr uint32_t OFF_STG = OFF_STK + 64 * 256;      // staging log_alpha [64][128] f32
constexpr uint32_t OFF_STB = OFF_STG + 64 * 512;      // staging beta [64] f32
// The inverse's scratch aliases the staging buffers: the next chunk is staged
// only after the inverse is done.
constexpr uint32_t OFF_AS = OFF_STQ;                  // A [64][65] f32
constexpr uint32_t OFF_XS = OFF_AS + 64 * 65 * 4;     // 32 x 33 f32 inverse scratch
constexpr uint32_t OFF_TS = OFF_STG;                  // T [64][65] f32
constexpr uint32_t SMEM_USED = OFF_STB + 256;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;     // + alignment slack
static_assert(OFF_XS + 32 * 33 * 4 <= OFF_STG, "inverse scratch must fit the q/k staging");
static_assert(OFF_TS + 64 * 65 * 4 <= OFF_STB, "T must fit the g staging");

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

// Tensor maps of the inputs (built on the host for each call).
struct TmaMaps {
  CUtensorMap q, k, la;   // [N, H, 128] boxes {128, 1, 64}, no swizzle (staging rows)
  CUtensorMap v;          // [N, H, dv]  boxes {64, 1, 64}, 128-byte swizzle (MMA operand tile)
};

constexpr uint32_t kStageBytes = 64 * 256 * 2 + 64 * 512;   // q + k + log_alpha of one chunk
constexpr uint32_t kVBytes = 64 * 128;

// Issue the TMA loads of q, k, log_alpha for the chunk starting at packed row c0
// (one thread), and load beta (threads 0..63; invalid rows get 0).
__device__ __forceinline__ void stage_chunk(const PrefillParams &p, const TmaMaps &m,
                                            const SeqSpan &sp, int c0, int h, unsigned char *base,
                                            uint64_t *bar, int tid) {
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, kStageBytes);
    tma_load_3d(smem_u32(base + OFF_STQ), &m.q, 0, h, c0, bar);
    tma_load_3d(smem_u32(base + OFF_STK), &m.k, 0, h, c0, bar);
    tma_load_3d(smem_u32(base + OFF_STG), &m.la, 0, h, c0, bar);
  }
  if (tid < kC) {
    const int pos = c0 + tid;
    float *sb = reinterpret_cast<float *>(base + OFF_STB);
    sb[tid] = row_valid(p, sp, pos) ? p.beta[(size_t)pos * p.H + h] : 0.f;
  }
}

// TMA load of the V slice (64 rows x 64 columns) straight into its MMA tile.
__device__ __forceinline__ void stage_v(const TmaMaps &m, int c0, int h, int dv0,
                                        unsigned char *base, uint64_t *bar, int tid) {
  if (tid == 0) {
    mbar_arrive_expect_tx(bar, kVBytes);
    tma_load_3d(smem_u32(base + OFF_V), &m.v, dv0, h, c0, bar);
  }
}

using prep::store_row32;

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(PrefillParams p, const __grid_constant__ TmaMaps maps) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ __align__(8) uint64_t stage_bar;
  __shared__ __align__(8) uint64_t v_bar;
  __shared__ uint32_t valid_sh[2];      // validity bits of the chunk's 64 rows
  __shared__ uint32_t unsafe_sh[4];     // channels with exact-path key rows
  __shared__ int tfirst_sh[128];        // their first exact-path key row
  const prep::ExactRows xrows{unsafe_sh, tfirst_sh};
  __shared__ float decay_sh[kDK];      // e^{g_C} per key channel
  __shared__ float beta_sh[kC];
  __shared__ float part_sh[4][kDK];

  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *base = smem_raw + pad;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lr = tid & 127;          // TMEM lane of this thread
  const int wg = tid >> 7;           // column half
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

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
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    mbar_init(&stage_bar, 1);
    mbar_init(&v_bar, 1);
  }
  for (int e = tid; e < 64 * 8; e += kThreads) {
    const int r = 64 + (e >> 3), ch = e & 7;
    *reinterpret_cast<uint4 *>(base + OFF_TBM + row_tile_chunk(r, 0, ch, 192)) = make_uint4(0, 0, 0, 0);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = tmem_base_sh;
  const uint32_t my_cols = lane_base + (uint32_t)(wg * 32);   // + accumulator base column
  uint32_t phase = 0;
  bool ok = true;

  {   // initial state: thread owns row lr, columns wg*32 .. +31
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      v[j] = p.init_state ? p.init_state[(((size_t)b * H + h) * kDK + lr) * DV + dv0 + wg * 32 + j] : 0.f;
    tmem_st32(tm + my_cols + TM_S, v);
    tmem_st_wait();
  }

  const uint32_t sQKW = smem_u32(base + OFF_QKW), sKH = smem_u32(base + OFF_KH);
  const uint32_t sKT = smem_u32(base + OFF_KT), sTBM = smem_u32(base + OFF_TBM);
  const uint32_t sV = smem_u32(base + OFF_V), sSB = smem_u32(base + OFF_SB);
  const uint32_t sUB = smem_u32(base + OFF_UB);
  float *As = reinterpret_cast<float *>(base + OFF_AS);
  float *Ts = reinterpret_cast<float *>(base + OFF_TS);
  float *Xs = reinterpret_cast<float *>(base + OFF_XS);
  const float *stb = reinterpret_cast<const float *>(base + OFF_STB);

  if (sp.begin < sp.end) {
    stage_chunk(p, maps, sp, sp.begin, h, base, &stage_bar, tid);
    stage_v(maps, sp.begin, h, dv0, base, &v_bar, tid);
  }
  uint32_t chunk_idx = 0;

  for (int c0 = sp.begin; c0 < sp.end; c0 += kC, ++chunk_idx) {
    // validity of the chunk's rows (tail rows and pads enter as identity steps)
    if (tid < kC) {
      const unsigned bits = __ballot_sync(0xFFFFFFFFu, row_valid(p, sp, c0 + tid));
      if ((tid & 31) == 0) valid_sh[tid >> 5] = bits;
    }
    if (tid < 4) unsafe_sh[tid] = 0u;
    ok = __syncthreads_and(mbar_wait(&stage_bar, chunk_idx & 1, p.wait_cycles) || (note_timeout(p.site, 21), false));
    if (!ok) break;
    // ---- P1: decay products and operand tiles
    {
      prep::PrepTiles t;
      t.qg = base + OFF_QKW; t.qg_R = 192; t.qg_row0 = 64;
      t.kg = base + OFF_QKW; t.kg_R = 192; t.kg_row0 = 128;
      t.kh = base + OFF_KH;
      t.kt = base + OFF_KT;
      prep::decay_and_tiles(reinterpret_cast<const uint16_t *>(base + OFF_STQ),
                            reinterpret_cast<const uint16_t *>(base + OFF_STK),
                            reinterpret_cast<const float *>(base + OFF_STG), valid_sh, t, part_sh,
                            decay_sh, stb, beta_sh, xrows, tid);
    }
    fence_async_smem();
    __syncthreads();
    // ---- Gram: [Q G ; K G] (K e^{-g})^T
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 64, 0, 0);
      for (int s = 0; s < 8; ++s)
        mma_bf16(tm + TM_G, desc_kmajor(sQKW, 192, 64, s), desc_kmajor(sKH, 64, 0, s), id, s > 0);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, p.wait_cycles) || (note_timeout(p.site, 22), false));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // channels whose chunk decay is out of the factorised range: exact terms added
    // (K e^{-g} has been read by the Gram: its region stages the fix-up)
    if (prep::any_unsafe(unsafe_sh))
      prep::exact_gram_fixup<false>(tm + my_cols + TM_G, xrows, valid_sh,
                                    reinterpret_cast<const uint16_t *>(p.q),
                                    reinterpret_cast<const uint16_t *>(p.k), p.log_alpha, c0, h, H,
                                    reinterpret_cast<float *>(base + OFF_KH), tid);
    // ---- P3: M rows (lanes 0-63) -> TBM rows 128..191; beta * A rows (lanes 64-127) -> As
    prep::extract_gram(tm + my_cols + TM_G, base + OFF_TBM, 192, 128, As, beta_sh, tid);
    __syncthreads();
    // ---- P4: T = (I + A)^{-1};  T_b = T Diag(beta) -> TBM rows 0..63
    tri::unit_lower_inverse_64(As, Ts, Xs, tid);
    prep::pack_tb(Ts, beta_sh, base + OFF_TBM, 192, tid);
    fence_async_smem();
    __syncthreads();
    // the staging buffers are free: stream the next chunk's q, k, log_alpha, beta
    if (c0 + kC < sp.end) stage_chunk(p, maps, sp, c0 + kC, h, base, &stage_bar, tid);
    // V of this chunk must have landed; zero its invalid rows
    ok = __syncthreads_and(mbar_wait(&v_bar, chunk_idx & 1, p.wait_cycles) || (note_timeout(p.site, 23), false));
    if (!ok) break;
    if ((valid_sh[0] & valid_sh[1]) != 0xFFFFFFFFu) {
      for (int e = tid; e < kC * 8; e += kThreads) {
        const int r = e >> 3, ch = e & 7;
        if (!((valid_sh[r >> 5] >> (r & 31)) & 1u))
          *reinterpret_cast<uint4 *>(base + OFF_V + row_tile_chunk(r, 0, ch, kC)) = make_uint4(0, 0, 0, 0);
      }
      fence_async_smem();
      __syncthreads();
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
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, p.wait_cycles) || (note_timeout(p.site, 24), false));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // ---- P6: -W into QKW rows 0..63 (lane = channel); S -> bf16 tile; S *= e^{g_C}
    {
      const int c = lr;
      float v[32];
      tmem_ld32(tm + my_cols + TM_W, v);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        *reinterpret_cast<__nv_bfloat16 *>(base + OFF_QKW + row_tile_off(wg * 32 + j, c, 192)) =
            __float2bfloat16_rn(-v[j]);
      tmem_ld32(tm + my_cols + TM_S, v);
      store_row32(base + OFF_SB, 128, c, wg * 4, v);
      const float decay = decay_sh[c];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= decay;
      tmem_st32(tm + my_cols + TM_S, v);
      tmem_st_wait();
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    if (c0 + kC < sp.end) stage_v(maps, c0 + kC, h, dv0, base, &v_bar, tid);   // U_v read V
    // ---- [U ; (Q G) S] += [-W ; Q G] S
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 64, 0, 1);
      for (int s = 0; s < 8; ++s)
        mma_bf16(tm + TM_D1, desc_kmajor(sQKW, 192, 0, s), desc_mnmajor(sSB, 128, 0, s), id, 1);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, p.wait_cycles) || (note_timeout(p.site, 25), false));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // ---- P8: U (lanes 0-63) -> bf16 tile
    if ((warp & 3) < 2) {
      float v[32];
      tmem_ld32(tm + my_cols + TM_D1, v);
      store_row32(base + OFF_UB, 64, lr, wg * 4, v);
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
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, p.wait_cycles) || (note_timeout(p.site, 26), false));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // ---- P10: O (lanes 64-127) -> global
    if ((warp & 3) >= 2) {
      float v[32];
      tmem_ld32(tm + my_cols + TM_D1, v);
      const int r = lr - kC;
      const int pos = c0 + r;
      if (pos < sp.end) {
        const bool valid = p.mask == nullptr || p.mask[pos] != 0;
        uint16_t *orow = reinterpret_cast<uint16_t *>(p.o) + ((size_t)pos * H + h) * DV + dv0 + wg * 32;
#pragma unroll
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
    fence_before_sync();
    __syncthreads();
  }

  if (!ok) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_TIMEOUT);
    // let the product that timed out finish (bounded) before TMEM is released
    mbar_wait(&mma_bar, (phase - 1) & 1, p.wait_cycles);
  } else if (p.final_state) {
    float v[32];
    tmem_ld32(tm + my_cols + TM_S, v);
    float *dst = p.final_state + (((size_t)b * H + h) * kDK + lr) * DV + dv0 + wg * 32;
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, TM_COLS);
  }
}

}  // namespace

bool prefill_tc_supported(const PrefillParams &p, bool bf16) {
  return bf16 && p.dk == kDK && (p.dv % kNV) == 0 && p.chunk == kC && !p.gate_head;
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool encode_3d(CUtensorMap *map, CUtensorMapDataType dt, size_t esize, const void *ptr, int inner,
               int H, int N, int box_inner, CUtensorMapSwizzle swz) {
  auto fn = get_encode();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)H, (cuuint64_t)(N > 0 ? N : 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)inner * esize, (cuuint64_t)inner * esize * H};
  const cuuint32_t box[3] = {(cuuint32_t)box_inner, 1u, 64u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillParams &p, cudaStream_t s) {
  if (p.num_seqs == 0) return cudaSuccess;
  TmaMaps maps;
  if (!encode_3d(&maps.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.q, kDK, p.H, p.N, kDK,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_3d(&maps.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.k, kDK, p.H, p.N, kDK,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_3d(&maps.la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.log_alpha, kDK, p.H, p.N, kDK,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_3d(&maps.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.v, p.dv, p.H, p.N, kNV,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)p.num_seqs * p.H * (p.dv / kNV);
  prefill_tc_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace kda
