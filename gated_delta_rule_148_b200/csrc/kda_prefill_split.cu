// Two-kernel tensor-core prefill: the state-independent work of every chunk
// runs fully in parallel, the state pass runs once per (sequence, head, d_v
// slice) with one product group per chunk on its chain.
//   intra (persistent CTAs over the (chunk, head) items, all SMs):  Q G, K e^{g_C-g},
//     M = tril(Q G (K e^{-g})^T),
//     T_b = (I + beta tril(K G (K e^{-g})^T))^{-1} Diag(beta), W = T_b K G, U_v = T_b V,
//     P'' = -(K e^{g_C-g})^T W - Diag(1 - e^{g_C}),  R = Q G - M W
//   state pass (one CTA per sequence, head, 32 or 64 columns of d_v; chunks in order):
//     O = R S + M U_v;  S <- S + P'' S + (K e^{g_C-g})^T U_v
// The second line is the WY update S <- Diag(e^{g_C}) S + (K e^{g_C-g})^T (U_v - W S)
// and O = (Q G) S + M (U_v - W S) regrouped so that the chain carries one product
// group per chunk ("Kimi Linear's 75% KV cache cut ...", theclarity.today, fourth
// paragraph: chunks and the WY representation; "Kimi Linear wlasnie pokonal ...",
// remio.ai: blockwise algorithm with a diagonal-plus-low-rank transition).
//
// The intra kernel writes each (chunk, head) item to the workspace in the exact
// 128-byte- or 64-byte-swizzled shared-memory tile layouts the state pass
// consumes; the state pass streams items back with bulk loads into two
// alternating buffers.  Workspace per item (90 112 bytes):
//   [0, 32768)      P''          128 x 128 bf16 row tile (row = output key channel)
//   [32768, 49152)  K e^{g_C-g}  64 x 128 bf16 row tile
//   [49152, 65536)  U_v          64 rows x 128 bf16 as four 32-column blocks (64-byte swizzle)
//   [65536, 81920)  R            64 x 128 bf16 row tile
//   [81920, 90112)  M            64 x 64 bf16 row tile (R and M read as one 64 x 192 tile)
#include <climits>

#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "kda_tc.cuh"
#include "kda_tril_inv.cuh"
#include "kda_chunk_prep.cuh"

namespace kda {
namespace split {

using namespace tc;

constexpr int kC = 64, kDK = 128, kNV = 64;

// ---- item layout
constexpr uint32_t IT_P = 0, IT_KT = 32768, IT_UV = 49152, IT_R = 65536, IT_M = 81920;
constexpr uint32_t ITEM_BYTES = 90112;

// ---- workspace layout
__host__ __device__ inline size_t ws_spans_bytes(int B) { return ((size_t)B * 16 + 255) / 256 * 256; }
__host__ __device__ inline size_t ws_cbase_off(int B) { return ws_spans_bytes(B); }
__host__ __device__ inline size_t ws_items_off(int B) {
  return (ws_cbase_off(B) + (size_t)(B + 1) * 4 + 1023) / 1024 * 1024;
}
__host__ __device__ inline size_t max_chunks(int N, int B) { return (size_t)N / kC + (size_t)B; }
__host__ __device__ inline size_t ws_total(int N, int B, int H) {
  return ws_items_off(B) + max_chunks(N, B) * (size_t)H * ITEM_BYTES;
}

// ============================================================ chunk index
// chunk_base[b] = number of 64-row chunks of sequences 0..b-1 (spans after edge pads).
__global__ void __launch_bounds__(1024) chunk_index_kernel(PrefillParams p, const SeqSpan *spans,
                                                           int *cbase) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  if (device_error_latched(p.err)) return;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < p.num_seqs; b0 += 1024) {
    const int b = b0 + tid;
    int n = 0;
    if (b < p.num_seqs) n = (spans[b].end - spans[b].begin + kC - 1) / kC;
    int x = n;   // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
      int t = warp_tot[lane], u = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, u, o);
        if (lane >= o) u += y;
      }
      warp_tot[lane] = u - t;   // exclusive prefix of warp totals
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

// Row r (a K index) of an MN-major operand tile with NS bf16 columns; this
// thread's NS/2 values start at 16-byte chunk chunk0.  64-byte rows: chunk c of
// row r sits at c ^ ((r >> 1) & 3); 128-byte rows: at c ^ (r & 7).
template <int NS>
__device__ __forceinline__ void store_operand_row(unsigned char *tile, int r, int chunk0,
                                                  const float *v) {
#pragma unroll
  for (int j = 0; j < NS / 2; j += 8) {
    uint4 pk;
    pk.x = pack_bf16x2(v[j + 0], v[j + 1]);
    pk.y = pack_bf16x2(v[j + 2], v[j + 3]);
    pk.z = pack_bf16x2(v[j + 4], v[j + 5]);
    pk.w = pack_bf16x2(v[j + 6], v[j + 7]);
    const int c = chunk0 + (j >> 3);
    const uint32_t off = NS == 64 ? (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4))
                                  : (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
    *reinterpret_cast<uint4 *>(tile + off) = pk;
  }
}

// ============================================================ intra kernel (A)
// Persistent: about two CTAs per SM loop over the (chunk, head) items, so the
// TMEM allocation, barrier set-up and constant tiles are paid once per CTA.
// ~100 KB of shared memory lets two CTAs share an SM and hide each other's load
// and tensor-core latency.  q, k, log_alpha are read straight from global
// memory, V arrives by TMA; the item's tiles leave through shared memory with
// bulk stores.
constexpr int kThreadsA = 256;
constexpr uint32_t A_QK = 0;                        // [Q G | K G] 128 x 128 row tile; then [Q G | W]
constexpr uint32_t A_KH = A_QK + 128 * 256;         // K e^{-g} 64 x 128; then A [64][65] f32; then U_v
constexpr uint32_t A_TB = A_KH + 17 * 1024;         // [T_b | 0]     128 x 64 row tile; then [M | 0]
constexpr uint32_t A_V = A_TB + 128 * 128;          // V  64 rows x 2 blocks of 64; then K e^{g_C-g}
constexpr uint32_t A_TS = A_V + 64 * 256;           // K e^{g_C-g} 64 x 128 tile; then T [64][65] f32
constexpr uint32_t A_XS = A_TS + 64 * 65 * 4;       // inverse scratch (32 x 33 f32)
constexpr uint32_t A_USED = A_XS + 32 * 33 * 4;
constexpr uint32_t A_SMEM = A_USED + 1024;
static_assert(A_TB % 1024 == 0 && A_V % 1024 == 0 && A_KH % 1024 == 0 && A_TS % 1024 == 0,
              "swizzled tiles are 1024-aligned");
static_assert(64 * 65 * 4 <= A_TB - A_KH, "A fits the K e^{-g} region");
constexpr uint32_t A_TM_GW = 0, A_TM_UV = 128, A_TM_COLS = 256;

__device__ __forceinline__ bool row_ok(const PrefillParams &p, const SeqSpan &sp, int pos) {
  return pos < sp.end && (p.mask == nullptr || p.mask[pos] != 0);
}

// Item -> (sequence, first row of its chunk, head): the sequence is the last b
// with cbase[b] <= the item's global chunk index.
struct ItemPos {
  int b, c0, h;
  size_t off;     // byte offset of the item in the workspace
};
__device__ __forceinline__ ItemPos locate_item(const PrefillParams &p, const SeqSpan *spans,
                                               const int *cbase, int item, int h0, int Hg) {
  const int gchunk = item / Hg;
  int lo = 0, hi = p.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cbase[mid] <= gchunk) lo = mid; else hi = mid - 1;
  }
  ItemPos ip;
  ip.b = lo;
  ip.h = h0 + item % Hg;
  ip.c0 = spans[lo].begin + (gchunk - cbase[lo]) * kC;
  ip.off = ((size_t)gchunk * p.H + ip.h) * ITEM_BYTES;
  return ip;
}

// Tensor maps of the intra kernel's inputs: V (loaded into its operand tile) and q, k,
// log_alpha (prefetched into L2 one item ahead; the prep reads them with plain loads).
struct IntraMaps {
  CUtensorMap v, q, k, la;
};

template <bool GATE_HEAD>     // log_alpha [N, H] (one gate per token and head) instead of [N, H, dk]
__global__ void __launch_bounds__(kThreadsA, 2)
intra_kernel(PrefillParams p, const __grid_constant__ IntraMaps maps, const SeqSpan *spans,
             const int *cbase, unsigned char *items, int h0, int Hg) {
  const CUtensorMap &vmap = maps.v;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ __align__(8) uint64_t v_bar;
  __shared__ __align__(8) uint64_t rl_bar;   // M and K e^{g_C-g} read back from the item
  __shared__ uint32_t valid_sh[2];
  __shared__ uint32_t unsafe_sh[4];     // channels whose Gram terms take the exact path
  __shared__ float decay_sh[kDK];
  __shared__ float beta_sh[kC];
  __shared__ float part_sh[4][kDK];

  if (device_error_latched(p.err)) return;
  const int H = p.H;
  const int nitems = cbase[p.num_seqs] * Hg;
  if ((int)blockIdx.x >= nitems) return;

  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *base = smem_raw + pad;
  const int tid = threadIdx.x, warp = tid >> 5, lr = tid & 127, wg = tid >> 7;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

  if (warp == 0) tmem_alloc(&tmem_base_sh, A_TM_COLS);
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    mbar_init(&v_bar, 1);
    mbar_init(&rl_bar, 1);
  }
  for (int e = tid; e < 64 * 8; e += kThreadsA) {     // rows 64..127 of [T_b | 0] = 0, for good
    const int r = 64 + (e >> 3), ch = e & 7;
    *reinterpret_cast<uint4 *>(base + A_TB + row_tile_chunk(r, 0, ch, 128)) = make_uint4(0, 0, 0, 0);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = tmem_base_sh;
  const uint32_t my_cols = lane_base + (uint32_t)(wg * 32);
  const uint32_t sQK = smem_u32(base + A_QK), sKH = smem_u32(base + A_KH);
  const uint32_t sTB = smem_u32(base + A_TB), sV = smem_u32(base + A_V);
  uint32_t phase = 0, vphase = 0, rphase = 0;
  bool ok = true;

  // V of an item is requested as soon as the previous item's products have read
  // the V tile, so its copy overlaps that item's read-out and stores.
  if (tid == 0 && (int)blockIdx.x < nitems) {
    const ItemPos ip = locate_item(p, spans, cbase, blockIdx.x, h0, Hg);
    mbar_arrive_expect_tx(&v_bar, 2 * 64 * 128);
    tma_load_3d(sV, &vmap, 0, ip.h, ip.c0, &v_bar);
    tma_load_3d(sV + 64 * 128, &vmap, 64, ip.h, ip.c0, &v_bar);
  }
  bool first = true;
  for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
    const ItemPos ip = locate_item(p, spans, cbase, item, h0, Hg);
    const int h = ip.h, c0 = ip.c0;
    const SeqSpan sp = spans[ip.b];
    unsigned char *it = items + ip.off;
    if (tid == 0 && item + (int)gridDim.x < nitems) {   // next item's q, k, log_alpha into L2
      const ItemPos nx = locate_item(p, spans, cbase, item + gridDim.x, h0, Hg);
      tma_prefetch_3d(&maps.q, 0, nx.h, nx.c0);
      tma_prefetch_3d(&maps.k, 0, nx.h, nx.c0);
      if (!GATE_HEAD) tma_prefetch_3d(&maps.la, 0, nx.h, nx.c0);
    }

    float beta_val = 0.f;      // stored to shared memory inside the prep, after its loads
    if (tid < kC) {
      const bool vr = row_ok(p, sp, c0 + tid);
      const unsigned bits = __ballot_sync(0xFFFFFFFFu, vr);
      if ((tid & 31) == 0) valid_sh[tid >> 5] = bits;
      if (vr) beta_val = __ldg(p.beta + (size_t)(c0 + tid) * H + h);
    }
    if (tid < 4) unsafe_sh[tid] = 0u;
    __syncthreads();
    // ---- decay products and operand tiles (global loads; V is already on its way)
    {
      prep::PrepTiles t;
      t.qg = base + A_QK; t.qg_R = 128; t.qg_row0 = 0;
      t.kg = base + A_QK; t.kg_R = 128; t.kg_row0 = 64;
      t.kh = base + A_KH;
      t.kt = nullptr;
      prep::decay_and_tiles_global<GATE_HEAD>(
          reinterpret_cast<const uint16_t *>(p.q), reinterpret_cast<const uint16_t *>(p.k), p.log_alpha,
          c0, h, H, valid_sh, t, nullptr, base + A_TS, nullptr, part_sh, decay_sh, beta_val, beta_sh,
          unsafe_sh, tid, !first);
    }
    fence_async_smem();
    __syncthreads();
    // ---- Gram: [Q G ; K G] (K e^{-g})^T  -> M (lanes 0-63), A / beta (lanes 64-127);
    //      K e^{g_C-g} leaves for the item
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_bf16(tm + A_TM_GW, desc_kmajor(sQK, 128, 0, s), desc_kmajor(sKH, 64, 0, s), id, s > 0);
      mma_commit(&mma_bar);
      bulk_store(it + IT_KT, base + A_TS, 64 * 256);
      bulk_commit();
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, p.wait_cycles));
    phase++;
    if (!ok) break;
    fence_after_sync();
    if (prep::any_unsafe(unsafe_sh))     // K e^{-g} is no longer needed: its region stages the fix-up
      prep::exact_gram_fixup<GATE_HEAD>(tm + my_cols + A_TM_GW, unsafe_sh, valid_sh,
                                        reinterpret_cast<const uint16_t *>(p.q),
                                        reinterpret_cast<const uint16_t *>(p.k), p.log_alpha, c0, h, H,
                                        reinterpret_cast<float *>(base + A_KH), tid);
    float *As = reinterpret_cast<float *>(base + A_KH);     // K e^{-g} is no longer needed
    float *Ts = reinterpret_cast<float *>(base + A_TS);
    float *Xs = reinterpret_cast<float *>(base + A_XS);
    {
      float v[32];
      tmem_ld32(tm + my_cols + A_TM_GW, v);
      if (lr < kC) {      // M row -> item (64 x 64 row tile), columns 32 wg .. 32 wg + 31
        const int r = lr;
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (wg * 32 + j <= r) ? v[j] : 0.f;
        prep::store_row32(it + IT_M, 64, r, wg * 4, v);
        asm volatile("fence.proxy.async.global;" ::: "memory");   // read back by a bulk copy
      } else {
        const int r = lr - kC;
        const float br = beta_sh[r];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int i = wg * 32 + j;
          As[r * 65 + i] = (i < r) ? br * v[j] : 0.f;
        }
      }
    }
    if (tid == 0) bulk_wait_read();     // K e^{g_C-g} has left the T region
    __syncthreads();
    tri::unit_lower_inverse_64(As, Ts, Xs, tid);
    prep::pack_tb(Ts, beta_sh, base + A_TB, 128, tid);
    fence_async_smem();
    ok = __syncthreads_and(mbar_wait(&v_bar, vphase & 1, p.wait_cycles));
    vphase++;
    if (!ok) break;
    // zero V rows of invalid positions (tail of the sequence, pads)
    if ((valid_sh[0] & valid_sh[1]) != 0xFFFFFFFFu) {
      for (int e = tid; e < kC * 16; e += kThreadsA) {
        const int r = e >> 4, blk = (e >> 3) & 1, ch = e & 7;
        if (!((valid_sh[r >> 5] >> (r & 31)) & 1u))
          *reinterpret_cast<uint4 *>(base + A_V + row_tile_chunk(r, blk, ch, kC)) = make_uint4(0, 0, 0, 0);
      }
      fence_async_smem();
      __syncthreads();
    }
    // ---- [W ; 0] = [T_b ; 0] (K G) ;  [U_v ; 0] = [T_b ; 0] V   (N = 128 each)
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + A_TM_GW, desc_kmajor(sTB, 128, 0, s), desc_mnmajor(sQK, 128, 64, s), id, s > 0);
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + A_TM_UV, desc_kmajor(sTB, 128, 0, s), desc_mnmajor(sV, 64, 0, s), id, s > 0);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, p.wait_cycles));
    phase++;
    if (!ok) break;
    fence_after_sync();
    // M and K e^{g_C-g} come back from the item (in L2) into the T_b and V tiles, whose
    // products are done, as the A operands of the last group
    if (tid == 0) {
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // the K e^{g_C-g} store is complete
      mbar_arrive_expect_tx(&rl_bar, 8192 + 16384);
      bulk_load(base + A_TB, it + IT_M, 8192, &rl_bar);
      bulk_load(base + A_V, it + IT_KT, 16384, &rl_bar);
    }
    if ((warp & 3) < 2) {
      // rows r = lr (< 64), columns 64 wg .. 64 wg + 63: W -> rows 64..127 of the Q G | K G
      // tile (K G is done; Q G stays for R), U_v -> the K e^{-g} region as 32-column blocks
      const int r = lr;
      float v[32];
      for (int q2 = 0; q2 < 2; ++q2) {
        tmem_ld32(tm + lane_base + A_TM_GW + (uint32_t)(wg * 64 + q2 * 32), v);
        prep::store_row32(base + A_QK + wg * 128 * 128, 128, 64 + r, q2 * 4, v);
        tmem_ld32(tm + lane_base + A_TM_UV + (uint32_t)(wg * 64 + q2 * 32), v);
        unsigned char *blk = base + A_KH + (2 * wg + q2) * 4096;
        store_operand_row<32>(blk, r, 0, v);
        store_operand_row<32>(blk, r, 2, v + 16);
      }
    }
    fence_async_smem();
    fence_before_sync();
    ok = __syncthreads_and(mbar_wait(&rl_bar, rphase & 1, p.wait_cycles));
    rphase++;
    if (!ok) break;
    // ---- P' = (K e^{g_C-g})^T W  (lanes = key channel);  [M W ; 0] = [M ; 0] W;  U_v -> item
    if (tid == 0) {
      fence_after_sync();
      bulk_store(it + IT_UV, base + A_KH, 64 * 256);
      bulk_commit();       // the next item's prep waits for this read before it rewrites the tiles
      const uint32_t idk = idesc_bf16(128, 128, 1, 1), idm = idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + A_TM_GW, desc_mnmajor(sV, 64, 0, s), desc_mnmajor(sQK, 128, 64, s), idk, s > 0);
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma_bf16(tm + A_TM_UV, desc_kmajor(sTB, 128, 0, s), desc_mnmajor(sQK, 128, 64, s), idm, s > 0);
      mma_commit(&mma_bar);
    }
    ok = __syncthreads_and(mbar_wait(&mma_bar, phase & 1, p.wait_cycles));
    phase++;
    if (!ok) break;
    fence_after_sync();
    if (tid == 0 && item + (int)gridDim.x < nitems) {   // the V tile is free: next item's V
      const ItemPos nx = locate_item(p, spans, cbase, item + gridDim.x, h0, Hg);
      mbar_arrive_expect_tx(&v_bar, 2 * 64 * 128);
      tma_load_3d(sV, &vmap, 0, nx.h, nx.c0, &v_bar);
      tma_load_3d(sV + 64 * 128, &vmap, 64, nx.h, nx.c0, &v_bar);
    }
    {
      // P'' = -P' - Diag(1 - e^{g_C}): row c = lr, columns 64 wg ..; R = Q G - M W: rows lr < 64
      const int c = lr;
      const float dg = 1.f - decay_sh[c];
      float v[32];
      for (int q2 = 0; q2 < 2; ++q2) {
        const int col0 = wg * 64 + q2 * 32;
        tmem_ld32(tm + lane_base + A_TM_GW + (uint32_t)col0, v);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) v[jj] = (col0 + jj == c) ? -v[jj] - dg : -v[jj];
        prep::store_row32(it + IT_P + wg * 128 * 128, 128, c, q2 * 4, v);
        tmem_ld32(tm + lane_base + A_TM_UV + (uint32_t)col0, v);
        if (c < kC) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float qg = __bfloat162float(
                *reinterpret_cast<const __nv_bfloat16 *>(base + A_QK + row_tile_off(c, col0 + jj, 128)));
            v[jj] = qg - v[jj];
          }
          prep::store_row32(it + IT_R + wg * 64 * 128, 64, c, q2 * 4, v);
        }
      }
    }
    first = false;
  }
  if (!ok) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_TIMEOUT);
    mbar_wait(&v_bar, (vphase - 0) & 1, 20000);
    mbar_wait(&rl_bar, rphase & 1, 20000);
    if (phase > 0) mbar_wait(&mma_bar, (phase - 1) & 1, p.wait_cycles);
  }
  if (tid == 0) {
    bulk_commit();
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // item stores complete
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, A_TM_COLS);
  }
}

// ============================================================ state pass (B)
// One product group per chunk on the chain.  With P'' = -(K e^{g_C-g})^T W -
// Diag(1 - e^{g_C}) (from the intra kernel), the chunk's state update
//   S <- Diag(e^{g_C}) S + (K e^{g_C-g})^T (U_v - W S)
// is S <- S + P'' S + (K e^{g_C-g})^T U_v: one group of products accumulating into
// S in TMEM, reading only the bf16 copy of S.  The chunk's output
//   O = (Q G) S + M (U_v - W S) = R S + M U_v,   R = Q G - M W,
// is a second group on the same bf16 copy, off the chain: it runs while the next
// chunk's S is converted.  The diagonal 1 - e^{g_C} rides in P'' in bf16 (its
// rounding error, ~2^-9 of the forgotten part of S, decays with S).
//
// 8 compute warps + 1 producer warp.  The producer streams each chunk's item
// into one of two buffers once both product groups that read the buffer are
// done.  A CTA owns NS columns of d_v (64 or 32): columns of the state never
// mix, so narrower slices give more independent chains.  The bf16 copy of S is
// double-buffered (the output group of chunk j reads it while chunk j + 1
// writes the other one); so is the output accumulator in TMEM.
constexpr int kComputeThreadsB = 256;
constexpr int kThreadsB = kComputeThreadsB + 32;

template <int NS>
struct StateTiles {
  static_assert(NS == 64 || NS == 32, "state slice of 64 or 32 columns");
  static constexpr int kCols = NS / 2;                   // d_v columns per compute thread
  // one item buffer: P'' | K e^{g_C-g} | R | M | U_v slice; the [R | M] operand is read
  // with M = 128 rows, i.e. 8 KB past the start of M, so every buffer is 80 KB
  static constexpr uint32_t P = 0, KT = 32768, R = 49152, M = 65536, UV = 73728;
  static constexpr uint32_t UV_BYTES = 64u * NS * 2u;
  static constexpr uint32_t BUF = 81920;
  static constexpr uint32_t TX = 32768 + 16384 + 16384 + 8192 + UV_BYTES;
  static constexpr uint32_t SB = 2 * BUF;                // bf16 S, two buffers of 128 x NS
  static constexpr uint32_t SB_BYTES = 128u * NS * 2u;
  static constexpr uint32_t SMEM = SB + 2 * SB_BYTES + 1024;
  static constexpr uint32_t TM_S = 0, TM_O = NS;         // O double buffer at NS and 2 NS
  static constexpr uint32_t TM_COLS = NS == 64 ? 256 : 128;
  static_assert(UV + UV_BYTES <= BUF && M + 16384 <= BUF, "item parts fit one buffer");
};

// Descriptor of K-step s (tile rows 16 s .. 16 s + 15) of such a tile with R rows.
template <int NS>
__device__ __forceinline__ uint64_t desc_operand(uint32_t base, int R, int s) {
  if constexpr (NS == 64) return desc_mnmajor(base, R, 0, s);
  else return sdesc(base + (uint32_t)(16 * s * 64), (uint32_t)(R * 64), 512, 4);
}

// Descriptor of K-step s of U_v as stored in the item: 64 rows (the chunk's positions),
// 32-column blocks of 64-byte rows with the 64-byte swizzle, blocks 4 KB apart; any
// number of consecutive blocks reads as one MN-major operand.
__device__ __forceinline__ uint64_t desc_uv(uint32_t base, int s) {
  return sdesc(base + (uint32_t)(16 * s * 64), 4096u, 512u, 4u);
}

template <int W>
__device__ __forceinline__ void tmem_ldw(uint32_t taddr, float *v) {
  if constexpr (W == 32) tmem_ld32(taddr, v); else tmem_ld16(taddr, v);
}
template <int W>
__device__ __forceinline__ void tmem_stw(uint32_t taddr, const float *v) {
  if constexpr (W == 32) tmem_st32(taddr, v); else tmem_st16(taddr, v);
}

template <int NS>
__device__ __forceinline__ void load_item(unsigned char *buf, const unsigned char *it, int dv0,
                                          uint64_t *bar) {
  using T = StateTiles<NS>;
  mbar_arrive_expect_tx(bar, T::TX);
  bulk_load(buf + T::P, it + IT_P, 32768 + 16384, bar);              // P'' and K e^{g_C-g}
  bulk_load(buf + T::R, it + IT_R, 16384 + 8192, bar);               // R and M
  bulk_load(buf + T::UV, it + IT_UV + (dv0 >> 5) * 4096, T::UV_BYTES, bar);
}

__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" :: "n"(kComputeThreadsB) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

template <int NS>
__global__ void __launch_bounds__(kThreadsB, 1)
state_kernel(PrefillParams p, const SeqSpan *spans, const int *cbase, const unsigned char *items,
             int h0, int Hg) {
  using T = StateTiles<NS>;
  constexpr int kW = T::kCols;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t s_bar;        // the state group of a chunk has landed
  __shared__ __align__(8) uint64_t o_bar;        // the output group of a chunk has landed
  __shared__ __align__(8) uint64_t load_bar[2];
  __shared__ __align__(8) uint64_t free_bar[2];
  __shared__ int err_sh;

  if (device_error_latched(p.err)) return;
  const int tiles = p.dv / NS;
  const int tile = blockIdx.x % tiles;
  const int h = h0 + (blockIdx.x / tiles) % Hg;
  const int b = blockIdx.x / (tiles * Hg);
  const int dv0 = tile * NS;
  const int H = p.H, DV = p.dv;
  const SeqSpan sp = spans[b];
  const int nch = (sp.end - sp.begin + kC - 1) / kC;
  const int cb = cbase[b];

  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *base = smem_raw + pad;
  const int tid = threadIdx.x, warp = tid >> 5, lr = tid & 127, wg = (tid >> 7) & 1;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t my_cols = lane_base + (uint32_t)(wg * kW);

  if (warp == 0) tmem_alloc(&tmem_base_sh, T::TM_COLS);
  if (tid == 0) {
    mbar_init(&s_bar, 1);
    mbar_init(&o_bar, 1);
    mbar_init(&load_bar[0], 1);
    mbar_init(&load_bar[1], 1);
    mbar_init(&free_bar[0], 1);
    mbar_init(&free_bar[1], 1);
    err_sh = 0;
  }
  // the bytes of each buffer past its U_v slice are read as rows of the output group that
  // nothing uses; keep them finite
  for (uint32_t e = T::UV + T::UV_BYTES + 16u * tid; e < T::BUF; e += 16u * kThreadsB) {
    *reinterpret_cast<uint4 *>(base + e) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(base + T::BUF + e) = make_uint4(0, 0, 0, 0);
  }
  fence_async_smem();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = tmem_base_sh;

  if (warp == kComputeThreadsB / 32) {
    // ---------------- producer warp: item loads, two chunks ahead of the chain
    if ((tid & 31) == 0 && !(p.fault & FAULT_STARVE_STATE_LOADS)) {
      for (int j = 0; j < nch; ++j) {
        if (j >= 2 && !mbar_wait(&free_bar[j & 1], ((j - 2) >> 1) & 1, p.wait_cycles)) {
          atomicOr(p.err, ERR_BIT_TIMEOUT);
          break;
        }
        if (*reinterpret_cast<volatile int *>(&err_sh)) break;
        load_item<NS>(base + (j & 1) * T::BUF, items + ((size_t)(cb + j) * H + h) * ITEM_BYTES, dv0,
                      &load_bar[j & 1]);
      }
    }
  } else {
    // ---------------- compute warps
    {   // initial state: thread owns state row lr, columns wg kW .. wg kW + kW - 1 of the slice
      float v[kW];
#pragma unroll
      for (int j = 0; j < kW; ++j)
        v[j] = p.init_state ? p.init_state[(((size_t)b * H + h) * kDK + lr) * DV + dv0 + wg * kW + j] : 0.f;
      tmem_stw<kW>(tm + my_cols + T::TM_S, v);
      tmem_st_wait();
    }
    uint32_t ps = 0, po = 0;          // phases of s_bar and o_bar waited for
    uint32_t nissued = 0;             // chunks whose two product groups were issued
    bool ok = true;

    // output epilogue of chunk jj: rows 0-63 of its accumulator (lanes 0-63) -> o
    auto epilogue = [&](int jj) {
      if ((warp & 3) < 2) {
        const int pos = sp.begin + jj * kC + lr;
        float v[kW];
        tmem_ldw<kW>(tm + my_cols + T::TM_O + (uint32_t)((jj & 1) * NS), v);
        if (pos < sp.end) {
          const bool valid = p.mask == nullptr || p.mask[pos] != 0;
          uint16_t *orow = reinterpret_cast<uint16_t *>(p.o) + ((size_t)pos * H + h) * DV + dv0 + wg * kW;
#pragma unroll
          for (int q = 0; q < kW; q += 8) {
            uint4 pk;
            pk.x = valid ? pack_bf16x2(v[q + 0], v[q + 1]) : 0u;
            pk.y = valid ? pack_bf16x2(v[q + 2], v[q + 3]) : 0u;
            pk.z = valid ? pack_bf16x2(v[q + 4], v[q + 5]) : 0u;
            pk.w = valid ? pack_bf16x2(v[q + 6], v[q + 7]) : 0u;
            *reinterpret_cast<uint4 *>(orow + q) = pk;
          }
        }
      }
    };

    for (int j = 0; j < nch; ++j) {
      const uint32_t sbuf = smem_u32(base + (j & 1) * T::BUF);
      unsigned char *sbf = base + T::SB + (j & 1) * T::SB_BYTES;
      if (!mbar_wait(&load_bar[j & 1], (j >> 1) & 1, p.wait_cycles)) err_sh = 1;
      // ---- S -> bf16 copy (the operand of both groups)
      {
        float v[kW];
        tmem_ldw<kW>(tm + my_cols + T::TM_S, v);
        store_operand_row<NS>(sbf, lr, wg * (kW / 8), v);
      }
      fence_async_smem();
      fence_before_sync();
      compute_sync();
      if (*reinterpret_cast<volatile int *>(&err_sh)) { ok = false; break; }
      nissued++;
      if (tid == 0) {
        fence_after_sync();
        const uint32_t ssb = smem_u32(sbf);
        // state group: S += P'' S_bf + (K e^{g_C-g})^T U_v
        const uint32_t idp = idesc_bf16(128, NS, 0, 1), idk = idesc_bf16(128, NS, 1, 1);
#pragma unroll
        for (int s = 0; s < 8; ++s)
          mma_bf16(tm + T::TM_S, desc_kmajor(sbuf + T::P, 128, 0, s), desc_operand<NS>(ssb, 128, s), idp, 1);
#pragma unroll
        for (int s = 0; s < 4; ++s)
          mma_bf16(tm + T::TM_S, desc_mnmajor(sbuf + T::KT, 64, 0, s), desc_uv(sbuf + T::UV, s), idk, 1);
        mma_commit(&s_bar);
        // output group: O = [R | M] [S_bf ; U_v]  (rows 64-127 of the result are not used)
        const uint32_t dO = tm + T::TM_O + (uint32_t)((j & 1) * NS);
#pragma unroll
        for (int s = 0; s < 12; ++s)
          mma_bf16(dO, desc_kmajor(sbuf + T::R, 64, 0, s),
                   s < 8 ? desc_operand<NS>(ssb, 128, s) : desc_uv(sbuf + T::UV, s - 8), idp, s > 0);
        mma_commit(&o_bar);
      }
      // ---- previous chunk's output while this chunk's groups run
      if (j > 0) {
        if (!mbar_wait(&o_bar, po & 1, p.wait_cycles)) err_sh = 1;
        po++;
        fence_after_sync();
        if (tid == 0) mbar_arrive(&free_bar[(j - 1) & 1]);   // both groups that read it are done
        epilogue(j - 1);
      }
      if (!mbar_wait(&s_bar, ps & 1, p.wait_cycles)) err_sh = 1;
      ps++;
      fence_after_sync();
    }
    if (ok && nch > 0 && !*reinterpret_cast<volatile int *>(&err_sh)) {
      if (!mbar_wait(&o_bar, po & 1, p.wait_cycles)) err_sh = 1;
      po++;
      fence_after_sync();
      epilogue(nch - 1);
    }
    fence_before_sync();
    compute_sync();
    ok = ok && !*reinterpret_cast<volatile int *>(&err_sh);
    if (!ok) {
      if (tid == 0) {
        err_sh = 1;
        atomicOr(p.err, ERR_BIT_TIMEOUT);
        // groups issued but not waited for, then item loads never consumed, land before exit
        for (; ps < nissued; ++ps) mbar_wait(&s_bar, ps & 1, p.wait_cycles);
        for (; po < nissued; ++po) mbar_wait(&o_bar, po & 1, p.wait_cycles);
        for (int jj = 0; jj < nch; ++jj) mbar_wait(&load_bar[jj & 1], (jj >> 1) & 1, 20000);
      }
    } else if (p.final_state) {
      float v[kW];
      tmem_ldw<kW>(tm + my_cols + T::TM_S, v);
      float *dst = p.final_state + (((size_t)b * H + h) * kDK + lr) * DV + dv0 + wg * kW;
#pragma unroll
      for (int jj = 0; jj < kW; jj += 4)
        *reinterpret_cast<float4 *>(dst + jj) = make_float4(v[jj], v[jj + 1], v[jj + 2], v[jj + 3]);
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, T::TM_COLS);
  }
}

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

}  // namespace split

bool prefill_split_supported(const PrefillParams &p, bool bf16) {
  return bf16 && p.dk == split::kDK && p.dv == 128 && p.chunk == split::kC;
}

size_t prefill_split_workspace(int N, int B, int H) { return split::ws_total(N, B, H); }

namespace {

constexpr int kMaxDev = 64;

int num_sms() {
  static int n[kMaxDev] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  if (n[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    n[dev] = v;
  }
  return n[dev];
}

}  // namespace

// spans: B entries already written by the pre-pass; ws: workspace base.
cudaError_t launch_prefill_split(const PrefillParams &p, SeqSpan *spans, void *ws, cudaStream_t s) {
  using namespace split;
  if (p.num_seqs == 0) return cudaSuccess;
  unsigned char *w = static_cast<unsigned char *>(ws);
  int *cbase = reinterpret_cast<int *>(w + ws_cbase_off(p.num_seqs));
  unsigned char *items = w + ws_items_off(p.num_seqs);
  chunk_index_kernel<<<1, 1024, 0, s>>>(p, spans, cbase);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  IntraMaps maps;
  if (!encode_3d(&maps.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.v, p.dv, p.H, p.N, kNV,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_3d(&maps.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.q, kDK, p.H, p.N, kDK,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_3d(&maps.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.k, kDK, p.H, p.N, kDK,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorNotSupported;
  if (p.gate_head) maps.la = maps.q;      // not used: the head-wise gate is 4 bytes per row
  else if (!encode_3d(&maps.la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.log_alpha, kDK, p.H, p.N, kDK,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorNotSupported;
  auto intra = p.gate_head ? intra_kernel<true> : intra_kernel<false>;
  e = cudaFuncSetAttribute(intra, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A_SMEM);
  if (e != cudaSuccess) return e;
  // 32-column state slices while they fit one wave (more independent chains, shorter products);
  // 64-column slices once there are more chains than SMs (less work per column in total).
  const bool narrow = (size_t)p.num_seqs * p.H * (p.dv / 32) <= (size_t)num_sms();
  auto state = narrow ? state_kernel<32> : state_kernel<64>;
  const uint32_t smem_b = narrow ? StateTiles<32>::SMEM : StateTiles<64>::SMEM;
  e = cudaFuncSetAttribute(state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b);
  if (e != cudaSuccess) return e;
  const size_t items_max = max_chunks(p.N, p.num_seqs) * (size_t)p.H;
  if (items_max > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  const size_t gridA = items_max < (size_t)(2 * num_sms()) ? items_max : (size_t)(2 * num_sms());
  intra<<<(unsigned)gridA, kThreadsA, A_SMEM, s>>>(p, maps, spans, cbase, items, 0, p.H);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const unsigned gridB = (unsigned)p.num_seqs * p.H * (p.dv / (narrow ? 32 : 64));
  state<<<gridB, kThreadsB, smem_b, s>>>(p, spans, cbase, items, 0, p.H);
  return cudaGetLastError();
}

}  // namespace kda
