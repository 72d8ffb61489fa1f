// Tensor-core prefill with chunks of 128 or 256 rows.
//
// The pages' own design uses 256-token chunks with the WY representation
// ("Kimi Linear's 75% KV cache cut ...", theclarity.today, fourth paragraph);
// a longer chunk shortens the serial chain of the state pass by 2x or 4x.  The
// chunk-C quantities are built from the 64-row items of the intra kernel
// (kda_prefill_split.cu) by merging neighbours, not by forming e^{-g} over C
// rows: for two consecutive sub-chunks a, b of c rows each (decays relative to
// their own starts; W, Q G, K~ = K e^{g_C-g}, U_v, M, gamma = e^{g_C} as in the
// 64-row item) the chunk of 2c rows has
//   W   = [W_a ; W_b Diag(gamma_a) - E W_a],      E = W_b K~_a^T   (c x c)
//   Q G = [Q G_a ; Q G_b Diag(gamma_a)]
//   K~  = [K~_a Diag(gamma_b) ; K~_b]
//   U_v = [U_v,a ; U_v,b - E U_v,a]
//   M   = [[M_a, 0], [F, M_b]],                   F = Q G_b K~_a^T
//   gamma = gamma_a gamma_b,
// which follows from running the two sub-chunk steps
//   U = U_v - W S,  O = Q G S + M U,  S <- Diag(gamma) S + K~^T U
// one after the other and collecting the terms in the state at the start of
// a.  Every factor is a decay product over rows that lie in order (<= 1), so
// the merge is exact for any log alpha <= 0 up to bf16 rounding of the merged
// tiles.  128-row items merge again into 256-row items.
//
// The state pass for chunk C streams each item in 32 KB parts (one 128 x 128
// bf16 tile each) through a ring of shared-memory slots, in the order its
// products read them: the 2C/128 row blocks of [-W ; Q G] (first product
// group), then the C/128 row blocks of K~ and the nonzero 128 x 128 blocks of
// M (second group).  A 256-row item (352 KB) does not fit in shared memory;
// the ring keeps only the parts in flight.
//
// Item layout for chunk C (P = C / 128 blocks of 128 rows):
//   part i            -W rows 128 i ..            (i < P)     128 x 128 row tile
//   part P + i        Q G rows 128 i ..
//   part 2P + i       K~ rows 128 i ..
//   part 3P + i(i+1)/2 + k   M block (i, k), k <= i
//   then U_v: two 64-column blocks of C rows x 128 B (row tile with C rows), then
//   e^{g_C} (128 fp32).
#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace big {

using namespace tc;

constexpr int kDK = 128;
constexpr uint32_t kPart = 32768;

// The 64-row item of the intra kernel.
constexpr uint32_t I64_WQ = 0, I64_KT = 32768, I64_UV = 49152, I64_M = 65536, I64_GC = 73728;
constexpr uint32_t I64_BYTES = 74752;

template <int C>
struct Item {
  static_assert(C == 128 || C == 256, "chunk of 128 or 256 rows");
  static constexpr int P = C / 128;
  static constexpr int NM = P * (P + 1) / 2;
  static constexpr int PARTS = 3 * P + NM;
  __host__ __device__ static constexpr uint32_t W(int i) { return (uint32_t)i * kPart; }
  __host__ __device__ static constexpr uint32_t Q(int i) { return (uint32_t)(P + i) * kPart; }
  __host__ __device__ static constexpr uint32_t K(int i) { return (uint32_t)(2 * P + i) * kPart; }
  __host__ __device__ static constexpr uint32_t M(int i, int k) { return (uint32_t)(3 * P + i * (i + 1) / 2 + k) * kPart; }
  static constexpr uint32_t UV = (uint32_t)PARTS * kPart;
  static constexpr uint32_t GC = UV + (uint32_t)C * 256;
  static constexpr uint32_t BYTES = GC + 512;
};

// Input item of a merge of c-row chunks: layout offsets of its parts.
template <int c>
struct In;
template <>
struct In<64> {
  static constexpr uint32_t BYTES = I64_BYTES, GC = I64_GC, UV = I64_UV;
};
template <>
struct In<128> {
  static constexpr uint32_t BYTES = Item<128>::BYTES, GC = Item<128>::GC, UV = Item<128>::UV;
};

// ---- workspace: spans | chunk indices for 64, 128, 256 | region A | region B
__host__ __device__ inline size_t spans_bytes(int B) { return ((size_t)B * 16 + 255) / 256 * 256; }
__host__ __device__ inline size_t cb_off(int B, int which) {   // which: 0 = 64, 1 = 128, 2 = 256
  return spans_bytes(B) + (size_t)which * (((size_t)B + 1) * 4 + 15) / 16 * 16;
}
__host__ __device__ inline size_t max_chunks(int N, int B, int C) { return (size_t)N / C + (size_t)B; }
__host__ __device__ inline size_t region_a_off(int B) { return (cb_off(B, 3) + 1023) / 1024 * 1024; }
__host__ __device__ inline size_t region_a_bytes(int N, int B, int H, int C) {
  const size_t a = max_chunks(N, B, 64) * H * I64_BYTES;
  const size_t z = C == 256 ? max_chunks(N, B, 256) * H * Item<256>::BYTES : 0;
  return ((a > z ? a : z) + 1023) / 1024 * 1024;
}
__host__ __device__ inline size_t ws_total(int N, int B, int H, int C) {
  return region_a_off(B) + region_a_bytes(N, B, H, C) + max_chunks(N, B, 128) * H * Item<128>::BYTES;
}

// cbase[b] = number of C-row chunks of the sequences before b (spans after edge pads).
template <int C>
__global__ void __launch_bounds__(1024) index_kernel(PrefillParams p, const SeqSpan *spans, int *cbase) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  if (device_error_latched(p.err)) return;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int b0 = 0; b0 < p.num_seqs; b0 += 1024) {
    const int b = b0 + tid;
    const int n = b < p.num_seqs ? (spans[b].end - spans[b].begin + C - 1) / C : 0;
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

// ============================================================ merge
// One CTA per (chunk of 2c rows, head): reads the items of its two c-row
// sub-chunks and writes the merged item.  The last chunk of a sequence with an
// odd number of sub-chunks has no second sub-chunk: it is the first one padded
// with identity rows (zero tiles, gamma unchanged).
constexpr int kThreadsM = 256;

template <int c>
struct MergeSmem;
// c = 64: [-W_b ; Q G_b] (32 KB), K~_a (16 KB), -W_a as rows 0-63 of a 128-row tile (its
// two 8 KB halves at WA and WA + 16 KB), U_v,a (16 KB).  E (64 x 64) sits in the 8 KB hole
// between the halves of -W_a; as the A operand of a 128-row product its rows 64-127 read
// the second half of -W_a, which only feeds result rows that are not used.  About 89 KB,
// so two CTAs share an SM.
template <>
struct MergeSmem<64> {
  static constexpr uint32_t WQB = 0, KTA = 32768, WA = 49152, E = 57344, UVA = 73728;
  static constexpr uint32_t LOAD_TX = 32768 + 16384 + 8192 + 8192 + 16384;
  static constexpr uint32_t SMEM = 90112 + 1024;
};
template <>
struct MergeSmem<128> {  // -W_b, Q G_b, K~_a, -W_a, U_v,a, E
  static constexpr uint32_t WB = 0, QB = 32768, KA = 65536, WA = 98304, UVA = 131072, E = 163840;
  static constexpr uint32_t LOAD_TX = 5 * 32768;
  static constexpr uint32_t SMEM = 196608 + 1024;
};

// Byte ranges copied (or zeroed, src == nullptr) from the sub-chunk items into the merged
// item.  Every thread keeps eight 16-byte loads in flight before it stores them.
struct Seg {
  unsigned char *dst;
  const unsigned char *src;
  uint32_t bytes;
};
constexpr int kMaxSegs = 24;

__device__ __forceinline__ void copy_segments(const Seg *segs, int n, int tid) {
  uint32_t total = 0;
  for (int i = 0; i < n; ++i) total += segs[i].bytes >> 4;
  int sgi = 0;               // this thread's indices only grow: a cursor over the segments
  uint32_t seg0 = 0, seg1 = segs[0].bytes >> 4;
  for (uint32_t first = (uint32_t)tid; first < total; first += 8 * kThreadsM) {
    uint4 v[8];
    unsigned char *dst[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      dst[u] = nullptr;
      const uint32_t idx = first + (uint32_t)u * kThreadsM;
      if (idx >= total) continue;
      while (idx >= seg1) {
        seg0 = seg1;
        seg1 += segs[++sgi].bytes >> 4;
      }
      const uint32_t off = (idx - seg0) * 16;
      dst[u] = segs[sgi].dst + off;
      v[u] = segs[sgi].src ? __ldg(reinterpret_cast<const uint4 *>(segs[sgi].src + off))
                           : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (dst[u]) *reinterpret_cast<uint4 *>(dst[u]) = v[u];
  }
}

__device__ __forceinline__ void unpack8(uint4 w, float *f) {
  const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(x[e] << 16);
    f[2 * e + 1] = __uint_as_float(x[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint4 pack8(const float *f) {
  uint4 w;
  w.x = pack_bf16x2(f[0], f[1]);
  w.y = pack_bf16x2(f[2], f[3]);
  w.z = pack_bf16x2(f[4], f[5]);
  w.w = pack_bf16x2(f[6], f[7]);
  return w;
}

// Row r, 64-column block kb of a row tile: dst = bf16(src * scale[col]) (+ add[] if given),
// 8 chunks of 8 columns; src/dst row tiles with Rs / Rd rows (row indices rs / rd).
__device__ __forceinline__ void scale_row(unsigned char *dst, int rd, int Rd, const unsigned char *src,
                                          int rs, int Rs, int kb, const float *scale, const float *add) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4 *>(src + row_tile_chunk(rs, kb, ch, Rs)), f);
    const float4 s0 = *reinterpret_cast<const float4 *>(scale + kb * 64 + ch * 8);
    const float4 s1 = *reinterpret_cast<const float4 *>(scale + kb * 64 + ch * 8 + 4);
    const float sc[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = f[e] * sc[e] + (add ? add[ch * 8 + e] : 0.f);
    *reinterpret_cast<uint4 *>(dst + row_tile_chunk(rd, kb, ch, Rd)) = pack8(f);
  }
}

// Row r, block kb: dst = bf16(src + add[]) (U_v rows).
__device__ __forceinline__ void add_row(unsigned char *dst, int rd, int Rd, const unsigned char *src,
                                        int rs, int Rs, int kb, const float *add) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {
    float f[8];
    unpack8(*reinterpret_cast<const uint4 *>(src + row_tile_chunk(rs, kb, ch, Rs)), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] += add[ch * 8 + e];
    *reinterpret_cast<uint4 *>(dst + row_tile_chunk(rd, kb, ch, Rd)) = pack8(f);
  }
}

template <int c>
__global__ void __launch_bounds__(kThreadsM, c == 64 ? 2 : 1)
merge_kernel(PrefillParams p, const SeqSpan *spans, const int *cb_in, const int *cb_out,
             const unsigned char *in, unsigned char *out) {
  using O = Item<2 * c>;
  using IN = In<c>;
  using SM = MergeSmem<c>;
  constexpr int RO = 2 * c;     // rows of the output's U_v tile
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t load_bar, mma_bar;
  __shared__ __align__(16) float gam_a[kDK], gam_b[kDK];

  if (device_error_latched(p.err)) return;
  const int H = p.H;
  const int gch = blockIdx.x / H, h = blockIdx.x % H;
  if (gch >= cb_out[p.num_seqs]) return;
  int lo = 0, hi = p.num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cb_out[mid] <= gch) lo = mid; else hi = mid - 1;
  }
  const int b = lo, j = gch - cb_out[b];
  const int ia = cb_in[b] + 2 * j;
  const bool has_b = 2 * j + 1 < cb_in[b + 1] - cb_in[b];
  const unsigned char *xa = in + ((size_t)ia * H + h) * IN::BYTES;
  const unsigned char *xb = xa + (size_t)H * IN::BYTES;
  unsigned char *o = out + ((size_t)gch * H + h) * O::BYTES;
  const int tid = threadIdx.x;

  if (tid < kDK) {
    gam_a[tid] = reinterpret_cast<const float *>(xa + IN::GC)[tid];
    gam_b[tid] = has_b ? reinterpret_cast<const float *>(xb + IN::GC)[tid] : 1.f;
  }

  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *base = smem_raw + pad;
  const int warp = tid >> 5, r = (warp & 3) * 32 + (tid & 31), wg = warp >> 2;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  if (has_b) {
    // the operand tiles of the two product groups load while the copies below run
    if (warp == 0) tmem_alloc(&tmem_base_sh, 256);
    if (tid == 0) {
      mbar_init(&load_bar, 1);
      mbar_init(&mma_bar, 1);
      mbar_arrive_expect_tx(&load_bar, SM::LOAD_TX);
      if constexpr (c == 64) {
        bulk_load(base + SM::WQB, xb + I64_WQ, 32768, &load_bar);
        bulk_load(base + SM::KTA, xa + I64_KT, 16384, &load_bar);
        bulk_load(base + SM::WA, xa + I64_WQ, 8192, &load_bar);
        bulk_load(base + SM::WA + 16384, xa + I64_WQ + 16384, 8192, &load_bar);
        bulk_load(base + SM::UVA, xa + I64_UV, 16384, &load_bar);
      } else {
        bulk_load(base + SM::WB, xb + Item<128>::W(0), kPart, &load_bar);
        bulk_load(base + SM::QB, xb + Item<128>::Q(0), kPart, &load_bar);
        bulk_load(base + SM::KA, xa + Item<128>::K(0), kPart, &load_bar);
        bulk_load(base + SM::WA, xa + Item<128>::W(0), kPart, &load_bar);
        bulk_load(base + SM::UVA, xa + Item<128>::UV, kPart, &load_bar);
      }
    }
  }

  // ---- parts that are copies of a sub-chunk's parts (or zero rows)
  Seg sg[kMaxSegs];
  int n = 0;
  auto add = [&](unsigned char *dst, const unsigned char *src, uint32_t bytes) { sg[n++] = Seg{dst, src, bytes}; };
  if constexpr (c == 64) {
    for (int kb = 0; kb < 2; ++kb) {
      add(o + O::W(0) + kb * 16384, xa + I64_WQ + kb * 16384, 8192);            // -W_a
      add(o + O::Q(0) + kb * 16384, xa + I64_WQ + kb * 16384 + 8192, 8192);     // Q G_a
      add(o + O::UV + kb * 16384, xa + I64_UV + kb * 8192, 8192);               // U_v,a
    }
    add(o + O::M(0, 0), xa + I64_M, 8192);                                       // M_a
    add(o + O::M(0, 0) + 16384, nullptr, 8192);                                  // upper right
    if (has_b) {
      for (int kb = 0; kb < 2; ++kb)
        add(o + O::K(0) + kb * 16384 + 8192, xb + I64_KT + kb * 8192, 8192);    // K~_b
      add(o + O::M(0, 0) + 16384 + 8192, xb + I64_M, 8192);                     // M_b
    } else {
      for (int kb = 0; kb < 2; ++kb) {
        add(o + O::W(0) + kb * 16384 + 8192, nullptr, 8192);
        add(o + O::Q(0) + kb * 16384 + 8192, nullptr, 8192);
        add(o + O::K(0) + kb * 16384, xa + I64_KT + kb * 8192, 8192);
        add(o + O::K(0) + kb * 16384 + 8192, nullptr, 8192);
        add(o + O::UV + kb * 16384 + 8192, nullptr, 8192);
      }
      add(o + O::M(0, 0) + 8192, nullptr, 8192);
      add(o + O::M(0, 0) + 16384 + 8192, nullptr, 8192);
    }
  } else {
    add(o + O::W(0), xa + Item<128>::W(0), kPart);
    add(o + O::Q(0), xa + Item<128>::Q(0), kPart);
    add(o + O::M(0, 0), xa + Item<128>::M(0, 0), kPart);
    for (int kb = 0; kb < 2; ++kb)
      add(o + O::UV + kb * 32768, xa + Item<128>::UV + kb * 16384, 16384);
    if (has_b) {
      add(o + O::K(1), xb + Item<128>::K(0), kPart);
      add(o + O::M(1, 1), xb + Item<128>::M(0, 0), kPart);
    } else {
      add(o + O::W(1), nullptr, kPart);
      add(o + O::Q(1), nullptr, kPart);
      add(o + O::K(0), xa + Item<128>::K(0), kPart);
      add(o + O::K(1), nullptr, kPart);
      add(o + O::M(1, 0), nullptr, kPart);
      add(o + O::M(1, 1), nullptr, kPart);
      for (int kb = 0; kb < 2; ++kb) add(o + O::UV + kb * 32768 + 16384, nullptr, 16384);
    }
  }
  copy_segments(sg, n, tid);
  if (tid < kDK) reinterpret_cast<float *>(o + O::GC)[tid] = gam_a[tid] * gam_b[tid];
  if (!has_b) return;

  // ---- the merged rows: two product groups
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = tmem_base_sh;
  bool ok = mbar_wait(&load_bar, 0, p.wait_cycles);
  if (!ok) note_timeout(p.site, 31);
  ok = __syncthreads_and(ok);
  const bool loaded = ok;
  bool issued1 = false, issued2 = false;
  if (ok) {
    // [E ; F] = [-W_b ; Q G_b] K~_a^T  (E carries the sign of the stored -W_b)
    if (tid == 0) {
      fence_after_sync();
      if constexpr (c == 64) {
        const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
        for (int s = 0; s < 8; ++s)
          mma_bf16(tm, desc_kmajor(smem_u32(base + SM::WQB), 128, 0, s),
                   desc_kmajor(smem_u32(base + SM::KTA), 64, 0, s), id, s > 0);
      } else {
        const uint32_t id = idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          mma_bf16(tm, desc_kmajor(smem_u32(base + SM::WB), 128, 0, s),
                   desc_kmajor(smem_u32(base + SM::KA), 128, 0, s), id, s > 0);
          mma_bf16(tm + 128, desc_kmajor(smem_u32(base + SM::QB), 128, 0, s),
                   desc_kmajor(smem_u32(base + SM::KA), 128, 0, s), id, s > 0);
        }
      }
      mma_commit(&mma_bar);
    }
    issued1 = true;
    ok = mbar_wait(&mma_bar, 0, p.wait_cycles);
    if (!ok) note_timeout(p.site, 32);
    ok = __syncthreads_and(ok);
  }
  if (ok) {
    fence_after_sync();
    // E -> bf16 operand tile; F -> the merged M
    if constexpr (c == 64) {
      float v[32];
      tmem_ld32(tm + lane_base + (uint32_t)(wg * 32), v);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 pk = pack8(v + 8 * q);
        const uint32_t off = row_tile_chunk(r, 0, wg * 4 + q, 128);
        if (r < 64) *reinterpret_cast<uint4 *>(base + SM::E + off) = pk;
        else *reinterpret_cast<uint4 *>(o + O::M(0, 0) + off) = pk;
      }
    } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld32(tm + lane_base + (uint32_t)(wg * 64 + half * 32), v);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(base + SM::E + row_tile_chunk(r, wg, half * 4 + q, 128)) = pack8(v + 8 * q);
        tmem_ld32(tm + 128 + lane_base + (uint32_t)(wg * 64 + half * 32), v);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(o + O::M(1, 0) + row_tile_chunk(r, wg, half * 4 + q, 128)) = pack8(v + 8 * q);
      }
    }
    fence_async_smem();
    fence_before_sync();
    __syncthreads();
    // G1 = E (-W_a) and G2 = E U_v,a  (rows 0 .. c-1 of the results are used)
    if (tid == 0) {
      fence_after_sync();
      const uint32_t id = idesc_bf16(128, 128, 0, 1);
      if constexpr (c == 64) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t a = desc_kmajor(smem_u32(base + SM::E), 128, 0, s);
          mma_bf16(tm, a, desc_mnmajor(smem_u32(base + SM::WA), 128, 0, s), id, s > 0);
          mma_bf16(tm + 128, a, desc_mnmajor(smem_u32(base + SM::UVA), 64, 0, s), id, s > 0);
        }
      } else {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const uint64_t a = desc_kmajor(smem_u32(base + SM::E), 128, 0, s);
          mma_bf16(tm, a, desc_mnmajor(smem_u32(base + SM::WA), 128, 0, s), id, s > 0);
          mma_bf16(tm + 128, a, desc_mnmajor(smem_u32(base + SM::UVA), 128, 0, s), id, s > 0);
        }
      }
      mma_commit(&mma_bar);
    }
    issued2 = true;
    ok = mbar_wait(&mma_bar, 1, p.wait_cycles);
    if (!ok) note_timeout(p.site, 33);
    ok = __syncthreads_and(ok);
  }
  if (ok) {
    fence_after_sync();
    // The product group read E = (-W_b) K~_a^T, so G1 = E (-W_a) and G2 = E U_v,a give
    //   -W'_b = (-W_b) Diag(gamma_a) + G1   and   U'_v,b = U_v,b + G2.
    if (c == 128 || r < 64) {
      float g[64];
      tmem_ld32(tm + lane_base + (uint32_t)(wg * 64), g);
      tmem_ld32(tm + lane_base + (uint32_t)(wg * 64 + 32), g + 32);
      if constexpr (c == 64)
        scale_row(o + O::W(0), 64 + r, 128, base + SM::WQB, r, 128, wg, gam_a, g);
      else
        scale_row(o + O::W(1), r, 128, base + SM::WB, r, 128, wg, gam_a, g);
      tmem_ld32(tm + 128 + lane_base + (uint32_t)(wg * 64), g);
      tmem_ld32(tm + 128 + lane_base + (uint32_t)(wg * 64 + 32), g + 32);
      add_row(o + O::UV, c + r, RO, xb + IN::UV, r, c, wg, g);
    }
    if (c == 128 || r >= 64) {
      const int rr = c == 64 ? r - 64 : r;
      if constexpr (c == 64) {
        scale_row(o + O::Q(0), 64 + rr, 128, base + SM::WQB, 64 + rr, 128, wg, gam_a, nullptr);
        scale_row(o + O::K(0), rr, 128, base + SM::KTA, rr, 64, wg, gam_b, nullptr);
      } else {
        scale_row(o + O::Q(1), rr, 128, base + SM::QB, rr, 128, wg, gam_a, nullptr);
        scale_row(o + O::K(0), rr, 128, base + SM::KA, rr, 128, wg, gam_b, nullptr);
      }
    }
  } else if (tid == 0) {
    atomicOr(p.err, ERR_BIT_TIMEOUT);
    // loads and products in flight finish before shared and tensor memory are released
    if (!loaded) mbar_wait(&load_bar, 0, p.wait_cycles);
    if (issued2) mbar_wait(&mma_bar, 1, p.wait_cycles);
    else if (issued1) mbar_wait(&mma_bar, 0, p.wait_cycles);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tm, 256);
  }
}

// ============================================================ state pass
// One CTA per (sequence, head, 32 columns of d_v); 8 compute warps and a
// producer warp.  Per chunk: S -> bf16 operand; [-W ; Q G] S (2P products of
// M = 128) into a double-buffered accumulator while S is scaled by e^{g_C};
// U = U_v - W S -> bf16; then S += K~^T U and O += M U; the output epilogue of
// chunk j runs while chunk j+1's first group is in flight.  Item parts arrive
// through a ring of 32 KB slots; each slot is released by a tensor-core commit
// once the products reading it are done.
constexpr int kComputeThreads = 256;
constexpr int kThreadsS = kComputeThreads + 32;
constexpr int NS = 32, kW = 16;

// Ring parts per chunk, in the order they are read: the 2P row blocks of [-W ; Q G] (first
// product group), the slice's 64-column U_v block with e^{g_C} behind it (the decay of S and
// the U conversion), the P row blocks of K~ and the NM blocks of M (second group).  A chunk's
// first-group tiles take the slots its predecessor's last tiles and first-group tiles
// release, so they load a whole chunk step ahead.
template <int C>
struct Ring {
  static constexpr int P = C / 128;
  static constexpr int NSLOT = 6;
  static constexpr int STEP_PARTS = 1 + Item<C>::PARTS;
  static constexpr uint32_t SLOT = kPart + 1024;             // 32 KB tile (or U_v block + e^{g_C})
  static constexpr uint32_t GC_IN_SLOT = (uint32_t)C * 128;
  static constexpr uint32_t SB = NSLOT * SLOT;               // S: 128 rows x 64 B
  static constexpr uint32_t UB = SB + 128 * 64;              // U: C rows x 64 B
  static constexpr uint32_t SMEM = UB + (uint32_t)C * 64 + 1024;
  static_assert(GC_IN_SLOT + 512 <= SLOT, "U_v block and e^{g_C} share a slot");
  static constexpr uint32_t TM_S = 0, TM_D1 = NS;            // D1 buffers of 2P blocks of NS columns
  static constexpr uint32_t TM_COLS = C == 128 ? 256 : 512;
  static_assert(TM_D1 + 2 * 2 * P * NS <= TM_COLS, "tensor memory");
  static_assert(SMEM <= 232448 - 256, "shared memory");
};

__device__ __forceinline__ void store_row32(unsigned char *tile, int r, int chunk0, const float *v) {
#pragma unroll
  for (int j = 0; j < kW; j += 8) {
    const int cc = chunk0 + (j >> 3);
    *reinterpret_cast<uint4 *>(tile + r * 64 + ((cc ^ ((r >> 1) & 3)) << 4)) = pack8(v + j);
  }
}
// K-step s (16 rows) of a 32-column MN-major operand tile with 64-byte rows.
__device__ __forceinline__ uint64_t desc32(uint32_t base, int s) {
  return sdesc(base + (uint32_t)(16 * s * 64), 8192, 512, 4);
}
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" :: "n"(kComputeThreads) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

template <int C>
__global__ void __launch_bounds__(kThreadsS, 1)
state_kernel(PrefillParams p, const SeqSpan *spans, const int *cbase, const unsigned char *items) {
  using R = Ring<C>;
  using IT = Item<C>;
  constexpr int P = R::P, NSLOT = R::NSLOT, PARTS = IT::PARTS, SP = R::STEP_PARTS;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ __align__(8) uint64_t full_bar[NSLOT], free_bar[NSLOT];
  __shared__ int err_sh;

  if (device_error_latched(p.err)) return;
  const int tiles = p.dv / NS;
  const int tile = blockIdx.x % tiles;
  const int h = (blockIdx.x / tiles) % p.H;
  const int b = blockIdx.x / (tiles * p.H);
  const int dv0 = tile * NS;
  const int H = p.H, DV = p.dv;
  const SeqSpan sp = spans[b];
  const int nch = (sp.end - sp.begin + C - 1) / C;
  const int cb = cbase[b];

  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  unsigned char *base = smem_raw + pad;
  const int tid = threadIdx.x, warp = tid >> 5, lr = tid & 127, wg = (tid >> 7) & 1;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t my_cols = lane_base + (uint32_t)(wg * kW);
  const int uv_blk = dv0 >> 6;
  const int uv_c0 = ((dv0 & 63) >> 3) + wg * (kW / 8);

  if (warp == 0) tmem_alloc(&tmem_base_sh, R::TM_COLS);
  if (tid == 0) {
    mbar_init(&mma_bar, 1);
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&free_bar[i], 1);
    }
    err_sh = 0;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tm = tmem_base_sh;

  if (warp == kComputeThreads / 32) {
    // ---------------- producer: every part of every chunk through the ring, in reading order
    if ((tid & 31) == 0 && !(p.fault & FAULT_STARVE_STATE_LOADS)) {
      int t = 0;
      bool stop = false;
      for (int j = 0; j < nch && !stop; ++j) {
        const unsigned char *it = items + ((size_t)(cb + j) * H + h) * IT::BYTES;
        for (int qq = 0; qq < SP; ++qq, ++t) {
          const int q = qq < 2 * P ? qq : (qq == 2 * P ? -1 : qq - 1);   // item tile, or -1: U_v
          const int slot = t % NSLOT, use = t / NSLOT;
          if (use >= 1 && !mbar_wait(&free_bar[slot], (use - 1) & 1, p.wait_cycles)) {
            note_timeout(p.site, 14);
            atomicOr(p.err, ERR_BIT_TIMEOUT);
            stop = true;
            break;
          }
          if (*reinterpret_cast<volatile int *>(&err_sh)) { stop = true; break; }
          unsigned char *dst = base + (uint32_t)slot * R::SLOT;
          if (q < 0) {
            mbar_arrive_expect_tx(&full_bar[slot], R::GC_IN_SLOT + 512);
            bulk_load(dst, it + IT::UV + (uint32_t)uv_blk * C * 128, R::GC_IN_SLOT, &full_bar[slot]);
            bulk_load(dst + R::GC_IN_SLOT, it + IT::GC, 512, &full_bar[slot]);
          } else {
            mbar_arrive_expect_tx(&full_bar[slot], kPart);
            bulk_load(dst, it + (uint32_t)q * kPart, kPart, &full_bar[slot]);
          }
        }
      }
      // every load issued here has landed before the CTA exits
      for (int q = 1; q <= NSLOT && t - q >= 0; ++q) {
        const int tt = t - q;
        mbar_wait(&full_bar[tt % NSLOT], (tt / NSLOT) & 1, p.wait_cycles);
      }
    }
  } else {
    // ---------------- compute warps
    {
      float v[kW];
#pragma unroll
      for (int j = 0; j < kW; ++j)
        v[j] = p.init_state ? p.init_state[(((size_t)b * H + h) * kDK + lr) * DV + dv0 + wg * kW + j] : 0.f;
      tmem_st16(tm + my_cols + R::TM_S, v);
      tmem_st_wait();
    }
    const uint32_t sSB = smem_u32(base + R::SB), sUB = smem_u32(base + R::UB);
    uint32_t phase = 0;      // mma_bar waits done
    int commits = 0;         // mma_bar commits issued (thread 0)
    bool ok = true;

    auto slot_ready = [&](int t) -> bool {
      return mbar_wait(&full_bar[t % NSLOT], (t / NSLOT) & 1, p.wait_cycles);
    };
    auto slot_ptr = [&](int t) -> unsigned char * { return base + (uint32_t)(t % NSLOT) * R::SLOT; };

    // ring part of item tile q of chunk j, and of chunk j's U_v block
    auto tile_part = [&](int j, int q) { return j * SP + (q < 2 * P ? q : q + 1); };
    auto uv_part = [&](int j) { return j * SP + 2 * P; };
    float sv[kW];            // this thread's slice of S at the start of the current chunk

    auto begin_chunk = [&](int j) {
      tmem_ld16(tm + my_cols + R::TM_S, sv);
      store_row32(base + R::SB, lr, wg * (kW / 8), sv);
      fence_async_smem();
      fence_before_sync();
      compute_sync();
      if (tid == 0) {
        fence_after_sync();
        const uint32_t id = idesc_bf16(128, NS, 0, 1);
        bool good = !err_sh;
        for (int i = 0; i < 2 * P && good; ++i) {
          const int t = tile_part(j, i);
          if (!slot_ready(t)) { good = false; err_sh = 1; note_timeout(p.site, 11); break; }
          const uint64_t a0 = desc_kmajor(smem_u32(slot_ptr(t)), 128, 0, 0);
          const uint32_t d = tm + R::TM_D1 + (uint32_t)(((j & 1) * 2 * P + i) * NS);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            mma_bf16(d, a0 + (uint64_t)((((s >> 2) * 128 * 128) + (s & 3) * 32) >> 4), desc32(sSB, s), id, s > 0);
        }
        for (int i = 0; i < 2 * P; ++i) mma_commit(&free_bar[tile_part(j, i) % NSLOT]);
        mma_commit(&mma_bar);
        ++commits;
      }
    };

    if (nch > 0) begin_chunk(0);
    for (int j = 0; j < nch; ++j) {
      const int c0 = sp.begin + j * C;
      const uint32_t d1 = R::TM_D1 + (uint32_t)((j & 1) * 2 * P * NS);
      // U_v rows of this thread and e^{g_C}: S is scaled in TMEM while the first group runs
      // (the group reads the bf16 copy)
      if (!slot_ready(uv_part(j))) { err_sh = 1; note_timeout(p.site, 16); }
      unsigned char *uvs = slot_ptr(uv_part(j));
      uint4 uv[P][kW / 8];
#pragma unroll
      for (int i = 0; i < P; ++i)
#pragma unroll
        for (int q = 0; q < kW / 8; ++q)
          uv[i][q] = *reinterpret_cast<const uint4 *>(uvs + row_tile_chunk(128 * i + lr, 0, uv_c0 + q, C));
      {
        const float decay = reinterpret_cast<const float *>(uvs + R::GC_IN_SLOT)[lr];
#pragma unroll
        for (int jj = 0; jj < kW; ++jj) sv[jj] *= decay;
        tmem_st16(tm + my_cols + R::TM_S, sv);
      }
      // ---- U = U_v - W S -> bf16 operand
      if (!mbar_wait(&mma_bar, phase & 1, p.wait_cycles)) { err_sh = 1; note_timeout(p.site, 12); }
      phase++;
      fence_after_sync();
#pragma unroll
      for (int i = 0; i < P; ++i) {
        float v[kW];
        tmem_ld16(tm + my_cols + d1 + (uint32_t)(i * NS), v);
#pragma unroll
        for (int q = 0; q < kW / 8; ++q) {
          float f[8];
          unpack8(uv[i][q], f);
#pragma unroll
          for (int e = 0; e < 8; ++e) v[q * 8 + e] += f[e];
        }
        store_row32(base + R::UB, 128 * i + lr, wg * (kW / 8), v);
      }
      tmem_st_wait();
      fence_async_smem();
      fence_before_sync();
      compute_sync();
      if (tid == 0) mbar_arrive(&free_bar[uv_part(j) % NSLOT]);   // U_v block and e^{g_C} of chunk j read
      if (*reinterpret_cast<volatile int *>(&err_sh)) { ok = false; break; }
      // ---- S += K~^T U;  O += M U
      if (tid == 0) {
        fence_after_sync();
        const uint32_t ids = idesc_bf16(128, NS, 1, 1);
        const uint32_t ido = idesc_bf16(128, NS, 0, 1);
        bool good = true;
        for (int i = 0; i < P && good; ++i) {
          const int t = tile_part(j, 2 * P + i);
          if (!slot_ready(t)) { good = false; break; }
          const uint64_t as = desc_mnmajor(smem_u32(slot_ptr(t)), 128, 0, 0);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            mma_bf16(tm + R::TM_S, as + (uint64_t)((16 * s * 128) >> 4), desc32(sUB, 8 * i + s), ids, 1);
        }
        for (int i = 0; i < P && good; ++i)
          for (int k = 0; k <= i && good; ++k) {
            const int t = tile_part(j, 3 * P + i * (i + 1) / 2 + k);
            if (!slot_ready(t)) { good = false; break; }
            const uint64_t a0 = desc_kmajor(smem_u32(slot_ptr(t)), 128, 0, 0);
#pragma unroll
            for (int s = 0; s < 8; ++s)
              mma_bf16(tm + d1 + (uint32_t)((P + i) * NS),
                       a0 + (uint64_t)((((s >> 2) * 128 * 128) + (s & 3) * 32) >> 4),
                       desc32(sUB, 8 * k + s), ido, 1);
          }
        if (!good) { err_sh = 1; note_timeout(p.site, 11); }
        for (int q = 2 * P; q < PARTS; ++q) mma_commit(&free_bar[tile_part(j, q) % NSLOT]);
        mma_commit(&mma_bar);
        ++commits;
      }
      if (!mbar_wait(&mma_bar, phase & 1, p.wait_cycles)) { err_sh = 1; note_timeout(p.site, 13); }
      phase++;
      fence_after_sync();
      if (j + 1 < nch) begin_chunk(j + 1);
      // ---- O -> global
#pragma unroll
      for (int i = 0; i < P; ++i) {
        const int pos = c0 + 128 * i + lr;
        float v[kW];
        tmem_ld16(tm + my_cols + d1 + (uint32_t)((P + i) * NS), v);
        if (pos < sp.end) {
          const bool valid = p.mask == nullptr || p.mask[pos] != 0;
          uint16_t *orow = reinterpret_cast<uint16_t *>(p.o) + ((size_t)pos * H + h) * DV + dv0 + wg * kW;
#pragma unroll
          for (int jj = 0; jj < kW; jj += 8)
            *reinterpret_cast<uint4 *>(orow + jj) = valid ? pack8(v + jj) : make_uint4(0u, 0u, 0u, 0u);
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
        // products still in flight finish before the tensor memory is released
        for (int q = (int)phase; q < commits; ++q) mbar_wait(&mma_bar, (uint32_t)q & 1, p.wait_cycles);
      }
    } else if (p.final_state) {
      float v[kW];
      tmem_ld16(tm + my_cols + R::TM_S, v);
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
    tmem_dealloc(tm, R::TM_COLS);
  }
}

}  // namespace big

bool prefill_bigchunk_supported(const PrefillParams &p, bool bf16) {
  return bf16 && p.dk == big::kDK && p.dv == 128 && (p.chunk == 128 || p.chunk == 256);
}

size_t prefill_bigchunk_workspace(int N, int B, int H, int chunk) {
  return big::ws_total(N, B, H, chunk);
}

cudaError_t launch_prefill_bigchunk(const PrefillParams &p, SeqSpan *spans, void *ws, cudaStream_t s) {
  using namespace big;
  if (p.num_seqs == 0) return cudaSuccess;
  const int B = p.num_seqs, C = p.chunk;
  unsigned char *w = static_cast<unsigned char *>(ws);
  int *cb64 = reinterpret_cast<int *>(w + cb_off(B, 0));
  int *cb128 = reinterpret_cast<int *>(w + cb_off(B, 1));
  int *cb256 = reinterpret_cast<int *>(w + cb_off(B, 2));
  unsigned char *ra = w + region_a_off(B);
  unsigned char *rb = ra + region_a_bytes(p.N, B, p.H, C);
  cudaError_t e = launch_split_items(p, spans, cb64, ra, s);
  if (e != cudaSuccess) return e;
  index_kernel<128><<<1, 1024, 0, s>>>(p, spans, cb128);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t g128 = max_chunks(p.N, B, 128) * (size_t)p.H;
  if (g128 > 0x7FFFFFFFull) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(merge_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)MergeSmem<64>::SMEM);
  if (e != cudaSuccess) return e;
  merge_kernel<64><<<(unsigned)g128, kThreadsM, MergeSmem<64>::SMEM, s>>>(p, spans, cb64, cb128, ra, rb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int *cb = cb128;
  const unsigned char *items = rb;
  if (C == 256) {
    index_kernel<256><<<1, 1024, 0, s>>>(p, spans, cb256);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t g256 = max_chunks(p.N, B, 256) * (size_t)p.H;
    e = cudaFuncSetAttribute(merge_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)MergeSmem<128>::SMEM);
    if (e != cudaSuccess) return e;
    merge_kernel<128><<<(unsigned)g256, kThreadsM, MergeSmem<128>::SMEM, s>>>(p, spans, cb128, cb256, rb, ra);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cb = cb256;
    items = ra;
  }
  const unsigned grid = (unsigned)p.num_seqs * p.H * (p.dv / NS);
  if (C == 128) {
    e = cudaFuncSetAttribute(state_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Ring<128>::SMEM);
    if (e != cudaSuccess) return e;
    state_kernel<128><<<grid, kThreadsS, Ring<128>::SMEM, s>>>(p, spans, cb, items);
  } else {
    e = cudaFuncSetAttribute(state_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Ring<256>::SMEM);
    if (e != cudaSuccess) return e;
    state_kernel<256><<<grid, kThreadsS, Ring<256>::SMEM, s>>>(p, spans, cb, items);
  }
  return cudaGetLastError();
}

}  // namespace kda
