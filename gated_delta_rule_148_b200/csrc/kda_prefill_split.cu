// Two-kernel tensor-core prefill: the state-independent work of every chunk
// runs fully in parallel, the state pass runs once per (sequence, head, d_v
// slice).  Same chunk algebra as the fused kernel (kda_prefill_tc.cu):
//   intra (persistent CTAs over the (chunk, head) items, all SMs):  Q G, K e^{g_C-g},
//     M = tril(Q G (K e^{-g})^T),
//     T_b = (I + beta tril(K G (K e^{-g})^T))^{-1} Diag(beta), W = T_b K G, U_v = T_b V, e^{g_C}
//   state pass (one CTA per sequence, head, 32 or 64 columns of d_v; chunks in order):
//     U = U_v - W S;  O = (Q G) S + M U;  S <- Diag(e^{g_C}) S + (K e^{g_C-g})^T U
// ("Kimi Linear's 75% KV cache cut ...", theclarity.today, fourth paragraph:
// chunks and the WY representation; "Kimi Linear wlasnie pokonal ...",
// remio.ai: blockwise algorithm with a diagonal-plus-low-rank transition.)
//
// The intra kernel writes each (chunk, head) item to the workspace in the exact
// 128-byte-swizzled shared-memory tile layout the state pass consumes, with
// bulk (TMA) stores; the state pass streams items back with bulk loads into
// two alternating buffers.  Workspace per item (74 752 bytes):
//   [0, 32768)      [-W ; Q G]  128 x 128 bf16 row tile
//   [32768, 49152)  K e^{g_C-g}  64 x 128 bf16 row tile
//   [49152, 65536)  U_v          64 rows x 128 bf16, two 64-column blocks (MN-major tile)
//   [65536, 73728)  M            64 x 64 bf16 row tile
//   [73728, 74240)  e^{g_C}      128 fp32
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
constexpr uint32_t IT_WQ = 0, IT_KT = 32768, IT_UV = 49152, IT_M = 65536, IT_GC = 73728;
constexpr uint32_t ITEM_BYTES = 74752;

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

// ============================================================ intra kernel (A)
// Persistent: about two CTAs per SM loop over the (chunk, head) items, so the
// TMEM allocation, barrier set-up and constant tiles are paid once per CTA.
// ~100 KB of shared memory lets two CTAs share an SM and hide each other's load
// and tensor-core latency.  q, k, log_alpha and V arrive by TMA one item ahead
// (staged in tiles the current item no longer needs); the item's tiles leave
// through shared memory with bulk stores, U_v and M by direct stores.
constexpr int kThreadsA = 256;
constexpr uint32_t A_QK = 0;                        // [Q G | K G] 128 x 128 row tile; then [-W | .]
constexpr uint32_t A_KH = A_QK + 128 * 256;         // K e^{-g} 64 x 128; then A [64][65] f32; then U_v
constexpr uint32_t A_TB = A_KH + 17 * 1024;         // [T_b | 0]     128 x 64 row tile
constexpr uint32_t A_V = A_TB + 128 * 128;          // V  64 rows x 2 blocks of 64
constexpr uint32_t A_TS = A_V + 64 * 256;           // K e^{g_C-g} 64 x 128 tile; then T [64][65] f32
constexpr int kLDA = 68;                            // row stride of the A and T f32 tiles (16-byte rows)
constexpr uint32_t A_XS = A_TS + 64 * kLDA * 4;     // inverse scratch (32 x 33 f32)
constexpr uint32_t A_USED = A_XS + 32 * 33 * 4;
constexpr uint32_t A_SMEM = A_USED + 1024;
static_assert(A_TB % 1024 == 0 && A_V % 1024 == 0 && A_KH % 1024 == 0 && A_TS % 1024 == 0,
              "swizzled tiles are 1024-aligned");
static_assert(64 * kLDA * 4 <= A_TB - A_KH, "A fits the K e^{-g} region");
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

// Every thread waits on `bar` (bounded); true only if all of them saw the phase
// complete.  A thread that gave up records `code` as the timeout site.
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity, const PrefillParams &p,
                                         unsigned code) {
  const bool w = mbar_wait(bar, parity, p.wait_cycles);
  if (!w) note_timeout(p.site, code);
  return __syncthreads_and(w);
}

// Tensor maps of the intra kernel's inputs: V [N, H, dv] (64-column boxes, 128-byte
// swizzle, straight into its operand tile) and log_alpha, q, k [N, H, dk] (one item's
// 64 x 128 rows, no swizzle, staged for the decay prep).
struct IntraMaps {
  CUtensorMap v, la, q, k;
};

// The next item's inputs are loaded by TMA into tiles the current item no longer
// needs, so the prep reads them from shared memory: q into the K e^{g_C-g} / T tile
// and k into the K e^{-g} / A region once the inverse has read A and T_b is packed
// (U_v then leaves by direct stores, not through that region), log_alpha into the
// T_b and V tiles (32 KB) once the W and U_v products have read them.  V follows
// once the prep has read the staged rows.  (The plain per-thread
// loads this replaces were held up by the number of misses an SM keeps in flight.)
// With the head-wise gate (4 bytes of gate per row) log_alpha is read by plain loads and
// V has its tile from the start of the item; q and k are staged the same way.
template <bool GATE_HEAD>     // log_alpha [N, H] (one gate per token and head) instead of [N, H, dk]
__global__ void __launch_bounds__(kThreadsA, 2)
intra_kernel(PrefillParams p, const __grid_constant__ IntraMaps maps, const SeqSpan *spans,
             const int *cbase, unsigned char *items, int h0, int Hg) {
  constexpr bool kStage = !GATE_HEAD;     // log_alpha staged (q and k always are)
  const CUtensorMap &vmap = maps.v;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ __align__(8) uint64_t v_bar;
  __shared__ __align__(8) uint64_t in_bar;     // an item's staged inputs: q, k (and log_alpha)
  __shared__ uint32_t valid_sh[2];
  __shared__ uint32_t unsafe_sh[4];     // channels with exact-path key rows
  __shared__ int tfirst_sh[128];        // their first exact-path key row
  const prep::ExactRows xrows{unsafe_sh, tfirst_sh};
  __shared__ __align__(16) float decay_sh[kDK];   // written 16 bytes at a time by the prep
  __shared__ __align__(16) float beta_sh[kC];   // read 16 bytes at a time by pack_tb
  __shared__ __align__(16) float part_sh[8][kDK];   // per row group of the decay prep

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
    mbar_init(&in_bar, kStage ? 3 : 2);
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
  uint32_t phase = 0, vphase = 0, iphase = 0;
  bool ok = true;
  constexpr uint32_t kLaBytes = 64 * kDK * 4, kQkBytes = 64 * kDK * 2;
  static_assert(A_TB + kLaBytes <= A_TS, "staged log_alpha fits the T_b and V tiles");
  static_assert(kQkBytes <= A_TB - A_KH && kQkBytes <= A_XS - A_TS, "staged q, k fit their tiles");
  auto stage_q = [&](int hh, int cc) {
    mbar_arrive_expect_tx(&in_bar, kQkBytes);
    tma_load_3d(smem_u32(base + A_TS), &maps.q, 0, hh, cc, &in_bar);
  };
  auto stage_k = [&](int hh, int cc) {
    mbar_arrive_expect_tx(&in_bar, kQkBytes);
    tma_load_3d(sKH, &maps.k, 0, hh, cc, &in_bar);
  };
  auto stage_la = [&](int hh, int cc) {
    mbar_arrive_expect_tx(&in_bar, kLaBytes);
    tma_load_3d(sTB, &maps.la, 0, hh, cc, &in_bar);
  };

  // V of an item is requested as soon as the previous item's products have read
  // the V tile, so its copy overlaps that item's read-out and stores.
  if (tid == 0 && (int)blockIdx.x < nitems) {
    const ItemPos ip = locate_item(p, spans, cbase, blockIdx.x, h0, Hg);
    stage_q(ip.h, ip.c0);
    stage_k(ip.h, ip.c0);
    if (kStage) {
      stage_la(ip.h, ip.c0);
    } else {
      mbar_arrive_expect_tx(&v_bar, 2 * 64 * 128);
      tma_load_3d(sV, &vmap, 0, ip.h, ip.c0, &v_bar);
      tma_load_3d(sV + 64 * 128, &vmap, 64, ip.h, ip.c0, &v_bar);
    }
  }
  bool first = true;
  // An item's position, span, row validity and beta (rows tid < 64) are read one item
  // ahead, so the item starts without waiting on these global loads.  The sequence of
  // the last item looked up (its chunk range and span) stays in registers, so while the
  // items stay in one sequence their positions need no load at all; beta is loaded for
  // row min(c0 + tid, N - 1) (always in bounds) and masked by the row's validity only
  // where it is used, an item later, so no instruction here waits for a load.
  struct Ahead {
    ItemPos ip;
    SeqSpan sp;
    bool vr;
    float beta;     // not yet masked by vr
  };
  int seq_lo = 0, seq_hi = -1;      // global chunk range [seq_lo, seq_hi) of sequence seq_b
  int seq_b = 0;
  SeqSpan seq_sp{0, 0};
  auto read_ahead = [&](int item) {
    Ahead a;
    const int gchunk = item / Hg;
    if (gchunk < seq_lo || gchunk >= seq_hi) {
      a.ip = locate_item(p, spans, cbase, item, h0, Hg);
      seq_b = a.ip.b;
      seq_lo = cbase[seq_b];
      seq_hi = cbase[seq_b + 1];
      seq_sp = spans[seq_b];
    } else {
      a.ip.b = seq_b;
      a.ip.h = h0 + item % Hg;
      a.ip.c0 = seq_sp.begin + (gchunk - seq_lo) * kC;
      a.ip.off = ((size_t)gchunk * p.H + a.ip.h) * ITEM_BYTES;
    }
    a.sp = seq_sp;
    a.vr = tid < kC && row_ok(p, a.sp, a.ip.c0 + tid);
    a.beta = 0.f;
    if (tid < kC) a.beta = __ldg(p.beta + (size_t)min(a.ip.c0 + tid, p.N - 1) * H + a.ip.h);
    return a;
  };
  Ahead nx = read_ahead(blockIdx.x);
  for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
    const Ahead cur = nx;
    if (item + (int)gridDim.x < nitems) nx = read_ahead(item + gridDim.x);   // loads overlap this item
    const ItemPos ip = cur.ip;
    const int h = ip.h, c0 = ip.c0;
    unsigned char *it = items + ip.off;

    const float beta_val = cur.vr ? cur.beta : 0.f;   // stored to shared memory inside the prep
    if (tid < kC) {
      const unsigned bits = __ballot_sync(0xFFFFFFFFu, cur.vr);
      if ((tid & 31) == 0) valid_sh[tid >> 5] = bits;
    }
    if (tid < 4) unsafe_sh[tid] = 0u;
    ok = wait_all(&in_bar, iphase & 1, p, 4);
    iphase++;
    if (!ok) break;
    // ---- decay products and operand tiles (q, k from global memory; log_alpha staged or
    //      from global memory; V is already on its way or follows)
    {
      prep::PrepTiles t;
      t.qg = base + A_QK; t.qg_R = 128; t.qg_row0 = 0;
      t.kg = base + A_QK; t.kg_R = 128; t.kg_row0 = 64;
      t.kh = base + A_KH;
      t.kt = nullptr;
      prep::decay_and_tiles_global<GATE_HEAD>(
          reinterpret_cast<const uint16_t *>(p.q), reinterpret_cast<const uint16_t *>(p.k), p.log_alpha,
          c0, h, H, valid_sh, t, nullptr, base + A_TS, reinterpret_cast<float *>(it + IT_GC), part_sh,
          decay_sh, beta_val, beta_sh, xrows, tid, !first,
          kStage ? reinterpret_cast<const float *>(base + A_TB) : nullptr,
          reinterpret_cast<const uint16_t *>(base + A_TS), reinterpret_cast<const uint16_t *>(base + A_KH));
    }
    if (kStage) {
      // every thread read its staged rows before the prep's internal barrier: rows 64..127
      // of [T_b | 0] back to zero, V into its tile
      for (int e = tid; e < 64 * 8; e += kThreadsA) {
        const int r = 64 + (e >> 3), ch = e & 7;
        *reinterpret_cast<uint4 *>(base + A_TB + row_tile_chunk(r, 0, ch, 128)) = make_uint4(0, 0, 0, 0);
      }
      if (tid == 0) {
        fence_async_smem();
        mbar_arrive_expect_tx(&v_bar, 2 * 64 * 128);
        tma_load_3d(sV, &vmap, 0, h, c0, &v_bar);
        tma_load_3d(sV + 64 * 128, &vmap, 64, h, c0, &v_bar);
      }
    }
    fence_async_smem();
    __syncthreads();
    // ---- Gram: [Q G ; K G] (K e^{-g})^T  -> M (lanes 0-63), A / beta (lanes 64-127);
    //      Q G and K e^{g_C-g} leave for the item
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_bf16(tm + A_TM_GW, desc_kmajor(sQK, 128, 0, s), desc_kmajor(sKH, 64, 0, s), id, s > 0);
      mma_commit(&mma_bar);
      bulk_store(it + IT_WQ + 64 * 128, base + A_QK, 64 * 128);                   // Q G, block 0
      bulk_store(it + IT_WQ + 128 * 128 + 64 * 128, base + A_QK + 128 * 128, 64 * 128);  // block 1
      bulk_store(it + IT_KT, base + A_TS, 64 * 256);
      bulk_commit();
    }
    ok = wait_all(&mma_bar, phase & 1, p, 1);
    phase++;
    if (!ok) break;
    fence_after_sync();
    if (prep::any_unsafe(unsafe_sh))     // K e^{-g} is no longer needed: its region stages the fix-up
      prep::exact_gram_fixup<GATE_HEAD>(tm + my_cols + A_TM_GW, xrows, valid_sh,
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
      } else {
        const int r = lr - kC;
        const float br = beta_sh[r];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int i = wg * 32 + j;
          *reinterpret_cast<float4 *>(As + r * kLDA + i) =
              make_float4(i < r ? br * v[j] : 0.f, i + 1 < r ? br * v[j + 1] : 0.f,
                          i + 2 < r ? br * v[j + 2] : 0.f, i + 3 < r ? br * v[j + 3] : 0.f);
        }
      }
    }
    if (tid == 0) bulk_wait_read();     // K e^{g_C-g} has left the T region
    __syncthreads();
    tri::unit_lower_inverse_64<kLDA>(As, Ts, Xs, tid);
    prep::pack_tb<kLDA>(Ts, beta_sh, base + A_TB, 128, tid);
    fence_async_smem();
    ok = wait_all(&v_bar, vphase & 1, p, 2);
    vphase++;
    if (!ok) break;
    if (tid == 32 && item + (int)gridDim.x < nitems) {
      // T is packed and A is consumed: next item's q into the T tile, k into the A region
      // (from warp 1, so thread 0 goes straight on to the W and U_v products)
      fence_async_smem();
      stage_q(nx.ip.h, nx.ip.c0);
      stage_k(nx.ip.h, nx.ip.c0);
    }
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
    ok = wait_all(&mma_bar, phase & 1, p, 3);
    phase++;
    if (!ok) break;
    fence_after_sync();
    if (tid == 0 && item + (int)gridDim.x < nitems) {   // the T_b and V tiles are free
      if (kStage) {            // next item's log_alpha
        stage_la(nx.ip.h, nx.ip.c0);
      } else {                   // next item's V
        mbar_arrive_expect_tx(&v_bar, 2 * 64 * 128);
        tma_load_3d(sV, &vmap, 0, nx.ip.h, nx.ip.c0, &v_bar);
        tma_load_3d(sV + 64 * 128, &vmap, 64, nx.ip.h, nx.ip.c0, &v_bar);
      }
    }
    if ((warp & 3) < 2) {
      // rows r = lr (< 64), columns 64 wg .. 64 wg + 63: -W -> rows 0..63 of the Q G | K G
      // tile (its products are done), left by bulk store; U_v straight to the item
      const int r = lr;
      float v[32];
      for (int q2 = 0; q2 < 2; ++q2) {
        tmem_ld32(tm + lane_base + A_TM_GW + (uint32_t)(wg * 64 + q2 * 32), v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = -v[j];
        prep::store_row32(base + A_QK + wg * 128 * 128, 128, r, q2 * 4, v);
        tmem_ld32(tm + lane_base + A_TM_UV + (uint32_t)(wg * 64 + q2 * 32), v);
        prep::store_row32(it + IT_UV + wg * 64 * 128, 64, r, q2 * 4, v);
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      bulk_store(it + IT_WQ, base + A_QK, 64 * 128);                              // -W, block 0
      bulk_store(it + IT_WQ + 128 * 128, base + A_QK + 128 * 128, 64 * 128);      // -W, block 1
      bulk_commit();       // the next item's tile writes wait for these reads
    }
    first = false;
  }
  if (!ok) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_TIMEOUT);
    mbar_wait(&v_bar, (vphase - 0) & 1, 20000);
    mbar_wait(&in_bar, iphase & 1, 20000);
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
// 8 compute warps + 1 producer warp.  The producer streams each chunk's item
// into one of two buffers as soon as the products that read the buffer are
// done; the compute warps run the chain and synchronise among themselves on a
// named barrier.  The output accumulator is double-buffered in TMEM, so a
// chunk's output epilogue runs while the next chunk's first product is in
// flight.
//
// A CTA owns NS columns of d_v (64 or 32).  Columns of the state never mix in
// the recurrence, so narrower slices give more CTAs independent chains with
// shorter products and conversions.  The bf16 copies of S and U that feed the
// products are MN-major tiles of NS columns: 128-byte rows with the 128-byte
// swizzle for NS = 64, 64-byte rows with the 64-byte swizzle for NS = 32.
constexpr int kComputeThreadsB = 256;
constexpr int kThreadsB = kComputeThreadsB + 32;
constexpr uint32_t BUF_WQ = 0, BUF_KT = 32768, BUF_UV = 49152, BUF_M = 57344, BUF_GC = 65536;
constexpr uint32_t BUF_BYTES = 66560;
constexpr uint32_t BUF_TX = 32768 + 16384 + 8192 + 8192 + 512;
constexpr uint32_t B_BUF0 = 0, B_BUF1 = BUF_BYTES, B_SB = 2 * BUF_BYTES;

template <int NS>
struct StateTiles {
  static_assert(NS == 64 || NS == 32, "state slice of 64 or 32 columns");
  static constexpr int kCols = NS / 2;               // d_v columns per compute thread
  static constexpr uint32_t kRow = NS * 2;           // bytes per row of the S and U operand tiles
  static constexpr uint32_t UB = B_SB + 128 * kRow;  // S: 128 rows (d_k), U: 64 rows (chunk)
  static constexpr uint32_t SMEM = UB + 64 * kRow + 1024;
  static constexpr uint32_t TM_S = 0, TM_D1 = NS;    // D1 buffers at NS and 2 NS
  static constexpr uint32_t TM_COLS = NS == 64 ? 256 : 128;
};

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

// Descriptor of K-step s (tile rows 16 s .. 16 s + 15) of such a tile with R rows.
template <int NS>
__device__ __forceinline__ uint64_t desc_operand(uint32_t base, int R, int s) {
  if constexpr (NS == 64) return desc_mnmajor(base, R, 0, s);
  else return sdesc(base + (uint32_t)(16 * s * 64), (uint32_t)(R * 64), 512, 4);
}

template <int W>
__device__ __forceinline__ void tmem_ldw(uint32_t taddr, float *v) {
  if constexpr (W == 32) tmem_ld32(taddr, v); else tmem_ld16(taddr, v);
}
template <int W>
__device__ __forceinline__ void tmem_stw(uint32_t taddr, const float *v) {
  if constexpr (W == 32) tmem_st32(taddr, v); else tmem_st16(taddr, v);
}

__device__ __forceinline__ void load_item(unsigned char *buf, const unsigned char *it, int uv_blk,
                                          uint64_t *bar) {
  mbar_arrive_expect_tx(bar, BUF_TX);
  bulk_load(buf + BUF_WQ, it + IT_WQ, 32768, bar);
  bulk_load(buf + BUF_KT, it + IT_KT, 16384, bar);
  bulk_load(buf + BUF_UV, it + IT_UV + uv_blk * 8192, 8192, bar);
  bulk_load(buf + BUF_M, it + IT_M, 8192, bar);
  bulk_load(buf + BUF_GC, it + IT_GC, 512, bar);
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
  __shared__ __align__(8) uint64_t mma_bar;
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
  // the item's U_v comes in 64-column blocks: this slice's block and this thread's first chunk in it
  const int uv_blk = dv0 >> 6;
  const int uv_c0 = ((dv0 & 63) >> 3) + wg * (kW / 8);

  if (warp == 0) tmem_alloc(&tmem_base_sh, T::TM_COLS);
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    mbar_init(&load_bar[0], 1);
    mbar_init(&load_bar[1], 1);
    mbar_init(&free_bar[0], 1);
    mbar_init(&free_bar[1], 1);
    err_sh = 0;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = tmem_base_sh;

  if (warp == kComputeThreadsB / 32) {
    // ---------------- producer warp: item loads, two chunks ahead of the chain
    if ((tid & 31) == 0 && !(p.fault & FAULT_STARVE_STATE_LOADS)) {
      for (int j = 0; j < nch; ++j) {
        if (j >= 2 && !mbar_wait(&free_bar[j & 1], ((j - 2) >> 1) & 1, p.wait_cycles)) {
          note_timeout(p.site, 14);
          atomicOr(p.err, ERR_BIT_TIMEOUT);
          break;
        }
        if (*reinterpret_cast<volatile int *>(&err_sh)) break;
        load_item(base + ((j & 1) ? B_BUF1 : B_BUF0), items + ((size_t)(cb + j) * H + h) * ITEM_BYTES,
                  uv_blk, &load_bar[j & 1]);
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
    const uint32_t sSB = smem_u32(base + B_SB), sUB = smem_u32(base + T::UB);
    uint32_t phase = 0;
    bool ok = true;

    // Chunk j: S -> bf16 operand; [-W ; Q G] S into D1[j & 1]; then S *= e^{g_C}
    // while that product runs (it reads the bf16 copy, not S).  The TMEM store
    // is waited for before the product that accumulates into S is issued.
    auto begin_chunk = [&](int j) {
      unsigned char *buf = base + ((j & 1) ? B_BUF1 : B_BUF0);
      if (!mbar_wait(&load_bar[j & 1], (j >> 1) & 1, p.wait_cycles)) { err_sh = 1; note_timeout(p.site, 11); }
      float v[kW];
      tmem_ldw<kW>(tm + my_cols + T::TM_S, v);
      store_operand_row<NS>(base + B_SB, lr, wg * (kW / 8), v);
      fence_async_smem();
      fence_before_sync();
      compute_sync();
      if (tid == 0 && !err_sh) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, NS, 0, 1);
        const uint32_t d1 = tm + T::TM_D1 + (uint32_t)((j & 1) * NS);
        const uint64_t a0 = desc_kmajor(smem_u32(buf) + BUF_WQ, 128, 0, 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)
          mma_bf16(d1, a0 + (uint64_t)((((s >> 2) * 128 * 128) + (s & 3) * 32) >> 4),
                   desc_operand<NS>(sSB, 128, s), id, s > 0);
        mma_commit(&mma_bar);
      }
      const float decay = reinterpret_cast<const float *>(buf + BUF_GC)[lr];
#pragma unroll
      for (int jj = 0; jj < kW; ++jj) v[jj] *= decay;
      tmem_stw<kW>(tm + my_cols + T::TM_S, v);
    };

    if (nch > 0) begin_chunk(0);
    for (int j = 0; j < nch; ++j) {
      const int c0 = sp.begin + j * kC;
      unsigned char *buf = base + ((j & 1) ? B_BUF1 : B_BUF0);
      const uint32_t sbuf = smem_u32(buf);
      const uint32_t d1 = T::TM_D1 + (uint32_t)((j & 1) * NS);
      // operands of this chunk's conversions that do not depend on the product
      uint4 uv[kW / 8];
      bool o_valid = false;
      if ((warp & 3) < 2) {
#pragma unroll
        for (int q = 0; q < kW / 8; ++q)
          uv[q] = *reinterpret_cast<const uint4 *>(buf + BUF_UV + row_tile_chunk(lr, 0, uv_c0 + q, kC));
      } else {
        const int pos = c0 + lr - kC;
        o_valid = pos < sp.end && (p.mask == nullptr || p.mask[pos] != 0);
      }
      // ---- wait for [-W S ; (Q G) S]; U = U_v - W S (lanes 0-63) -> bf16 operand
      if (!mbar_wait(&mma_bar, phase & 1, p.wait_cycles)) { err_sh = 1; note_timeout(p.site, 12); }
      phase++;
      fence_after_sync();
      if ((warp & 3) < 2) {
        float v[kW];
        tmem_ldw<kW>(tm + my_cols + d1, v);
#pragma unroll
        for (int q = 0; q < kW / 8; ++q) {
          const uint32_t w[4] = {uv[q].x, uv[q].y, uv[q].z, uv[q].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            v[q * 8 + 2 * e] += __uint_as_float(w[e] << 16);
            v[q * 8 + 2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
          }
        }
        store_operand_row<NS>(base + T::UB, lr, wg * (kW / 8), v);
      }
      tmem_st_wait();      // S *= e^{g_C} has landed
      fence_async_smem();
      fence_before_sync();
      compute_sync();
      if (*reinterpret_cast<volatile int *>(&err_sh)) { ok = false; break; }
      // ---- O += [x ; M] U (rows 0-63 of the result are not used);  S += (K e^{g_C-g})^T U
      if (tid == 0) {
        fence_after_sync();
        const uint32_t ido = idesc_bf16(128, NS, 0, 1);
        const uint32_t ids = idesc_bf16(128, NS, 1, 1);
        const uint64_t ao = desc_kmajor(sbuf + BUF_UV, 128, 0, 0);
        const uint64_t as = desc_mnmajor(sbuf + BUF_KT, 64, 0, 0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
          mma_bf16(tm + d1, ao + (uint64_t)(s * 2), desc_operand<NS>(sUB, 64, s), ido, 1);
#pragma unroll
        for (int s = 0; s < 4; ++s)
          mma_bf16(tm + T::TM_S, as + (uint64_t)((16 * s * 128) >> 4), desc_operand<NS>(sUB, 64, s), ids, 1);
        mma_commit(&mma_bar);
      }
      if (!mbar_wait(&mma_bar, phase & 1, p.wait_cycles)) { err_sh = 1; note_timeout(p.site, 13); }
      phase++;
      fence_after_sync();
      if (tid == 0) mbar_arrive(&free_bar[j & 1]);     // the products that read buffer j & 1 are done
      // ---- next chunk's first product goes out before this chunk's output epilogue
      if (j + 1 < nch) begin_chunk(j + 1);
      // ---- O (lanes 64-127 of D1[j & 1]) -> global
      if ((warp & 3) >= 2) {
        const int r = lr - kC;
        const int pos = c0 + r;
        float v[kW];
        tmem_ldw<kW>(tm + my_cols + d1, v);
        if (pos < sp.end) {
          uint16_t *orow = reinterpret_cast<uint16_t *>(p.o) + ((size_t)pos * H + h) * DV + dv0 + wg * kW;
#pragma unroll
          for (int jj = 0; jj < kW; jj += 8) {
            uint4 pk;
            pk.x = o_valid ? pack_bf16x2(v[jj + 0], v[jj + 1]) : 0u;
            pk.y = o_valid ? pack_bf16x2(v[jj + 2], v[jj + 3]) : 0u;
            pk.z = o_valid ? pack_bf16x2(v[jj + 4], v[jj + 5]) : 0u;
            pk.w = o_valid ? pack_bf16x2(v[jj + 6], v[jj + 7]) : 0u;
            *reinterpret_cast<uint4 *>(orow + jj) = pk;
          }
        }
      }
    }
    tmem_st_wait();
    compute_sync();
    ok = ok && !*reinterpret_cast<volatile int *>(&err_sh);
    if (!ok) {
      if (tid == 0) {
        err_sh = 1;
        atomicOr(p.err, ERR_BIT_TIMEOUT);
      }
      if (phase > 0) mbar_wait(&mma_bar, (phase - 1) & 1, p.wait_cycles);
    } else if (p.final_state) {
      float v[kW];
      tmem_ldw<kW>(tm + my_cols + T::TM_S, v);
      float *dst = p.final_state + (((size_t)b * H + h) * kDK + lr) * DV + dv0 + wg * kW;
#pragma unroll
      for (int jj = 0; jj < kW; jj += 4)
        *reinterpret_cast<float4 *>(dst + jj) = make_float4(v[jj], v[jj + 1], v[jj + 2], v[jj + 3]);
    }
    if (tid == 0 && !ok) {
      // item loads the producer issued but the chain never consumed land before exit
      for (int jj = 0; jj < nch; ++jj) mbar_wait(&load_bar[jj & 1], (jj >> 1) & 1, 20000);
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

// The chunk index and the intra kernel: cbase[b] (b <= num_seqs) = 64-row chunks of the
// sequences before b; items = one 74 752-byte item per (64-row chunk, head).
cudaError_t launch_split_items(const PrefillParams &p, const SeqSpan *spans, int *cbase,
                               unsigned char *items, cudaStream_t s) {
  using namespace split;
  chunk_index_kernel<<<1, 1024, 0, s>>>(p, spans, cbase);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  IntraMaps maps;
  if (!encode_3d(&maps.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.v, p.dv, p.H, p.N, kNV,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  if (!encode_3d(&maps.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.q, kDK, p.H, p.N, kDK,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_3d(&maps.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.k, kDK, p.H, p.N, kDK,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorNotSupported;
  if (p.gate_head) {
    maps.la = maps.v;      // not used: the head-wise gate (4 bytes a row) is read by plain loads
  } else if (!encode_3d(&maps.la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.log_alpha, kDK, p.H, p.N, kDK,
                        CU_TENSOR_MAP_SWIZZLE_NONE)) {
    return cudaErrorNotSupported;
  }
  auto intra = p.gate_head ? intra_kernel<true> : intra_kernel<false>;
  e = cudaFuncSetAttribute(intra, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)A_SMEM);
  if (e != cudaSuccess) return e;
  const size_t items_max = max_chunks(p.N, p.num_seqs) * (size_t)p.H;
  if (items_max > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  const size_t gridA = items_max < (size_t)(2 * num_sms()) ? items_max : (size_t)(2 * num_sms());
  intra<<<(unsigned)gridA, kThreadsA, A_SMEM, s>>>(p, maps, spans, cbase, items, 0, p.H);
  return cudaGetLastError();
}

// spans: B entries already written by the pre-pass; ws: workspace base.
cudaError_t launch_prefill_split(const PrefillParams &p, SeqSpan *spans, void *ws, cudaStream_t s) {
  using namespace split;
  if (p.num_seqs == 0) return cudaSuccess;
  unsigned char *w = static_cast<unsigned char *>(ws);
  int *cbase = reinterpret_cast<int *>(w + ws_cbase_off(p.num_seqs));
  unsigned char *items = w + ws_items_off(p.num_seqs);
  cudaError_t e = launch_split_items(p, spans, cbase, items, s);
  if (e != cudaSuccess) return e;
  // 32-column state slices while they fit one wave (more independent chains, shorter products);
  // 64-column slices once there are more chains than SMs (less work per column in total).
  const bool narrow = (size_t)p.num_seqs * p.H * (p.dv / 32) <= (size_t)num_sms();
  auto state = narrow ? state_kernel<32> : state_kernel<64>;
  const uint32_t smem_b = narrow ? StateTiles<32>::SMEM : StateTiles<64>::SMEM;
  e = cudaFuncSetAttribute(state, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b);
  if (e != cudaSuccess) return e;
  const unsigned gridB = (unsigned)p.num_seqs * p.H * (p.dv / (narrow ? 32 : 64));
  state<<<gridB, kThreadsB, smem_b, s>>>(p, spans, cbase, items, 0, p.H);
  return cudaGetLastError();
}

}  // namespace kda
