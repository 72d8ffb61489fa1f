// Per-chunk intra work of the tensor-core prefill, shared by the fused kernel
// and the intra kernel of the two-kernel path.  All functions run on 256
// threads (two warpgroups); thread t owns TMEM lane t % 128 and the column half
// t / 128 of any 64-column accumulator it reads.
//
// Chunk algebra (C = 64 rows, g = inclusive per-channel cumsum of log_alpha in
// the chunk, a_r = e^{log_alpha_r}; "Kimi Linear's 75% KV cache cut ...",
// theclarity.today, fourth paragraph, WY form of a chunk):
//   e^{g_r} = prod_{j<=r} a_j,  e^{g_C - g_r} = prod_{j>r} a_j,  e^{-g_r} = e^{g_C - g_r} / e^{g_C}
//   Q G = q e^{g},  K G = k e^{g},  K e^{-g},  K e^{g_C - g}  (bf16 operand tiles)
//
// Range of the factorised Gram.  The Gram products take e^{g_r - g_i} as
// e^{g_r} * e^{-g_i}.  The factor e^{-g_i} of key row i and channel c is used
// only while e^{g_i} > kFastMinDecay (log-decay from the chunk start above about
// -60), where it is far from overflow; from the first row where it is not (the
// channel's threshold row t_c), the channel's K e^{-g} entries are 0 and
// exact_gram_fixup() adds those key rows' terms with running products of alpha
// on the CUDA cores (every factor <= 1, exact for any log_alpha <= 0).  Whether a
// key row takes the exact path depends on rows up to it only, so an output row
// never depends on a later row's values (prefix invariance, bit for bit).  A
// factor e^{g_r} that underflows multiplies terms below e^{-27} of the largest.
// The other tiles only use factors <= 1 and need no special case.
#pragma once

#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace prep {

using namespace tc;

constexpr int kC = 64;
constexpr int kDK = 128;
constexpr float kFastMinDecay = 1e-26f;   // e^{g_r} at or below this: exact path from row r on

// Per-chunk record of the exact-path key rows, in shared memory: bit c of `unsafe`
// (4 words, zeroed by the caller before the prep) is set when channel c has a
// threshold row, tfirst[c] (128 ints, set to 64 by the prep) is that row.
struct ExactRows {
  uint32_t *unsafe;
  int *tfirst;
};

// K e^{-g} entry of row r, channel c, from k and e^{g_r} (see the range note above);
// `marked` keeps the thread from recording the channel twice.
__device__ __forceinline__ float kh_entry(float k, float eg, int r, int c, const ExactRows &x,
                                          bool &marked) {
  if (eg > kFastMinDecay) {      // eg is a normal number here; the result is rounded to bf16
    float inv;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(eg));
    return k * inv;
  }
  if (!marked) {
    atomicMin(&x.tfirst[c], r);
    atomicOr(&x.unsafe[c >> 5], 1u << (c & 31));
    marked = true;
  }
  return 0.f;
}

template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

struct PrepTiles {
  unsigned char *qg;      // Q G rows (K-major row tile `qg_R` rows, starting row `qg_row0`)
  int qg_R, qg_row0;
  unsigned char *kg;      // K G rows (same tile as qg in both kernels)
  int kg_R, kg_row0;
  unsigned char *kh;      // K e^{-g}      (64-row tile)
  unsigned char *kt;      // K e^{g_C - g} (64-row tile)
};

// P1.  Thread: channels 2cp, 2cp+1 (cp = tid % 64), rows 16qt..16qt+15 (qt = tid / 64).
// Reads staged q, k ([64][128] bf16) and log_alpha ([64][128] f32); rows whose bit is
// clear in `valid` count as zero.  Writes the four operand tiles, decay[c] = e^{g_C}
// (qt == 0 threads) and beta_out (threads 0..63 copy beta_in).  Contains one
// __syncthreads(); must be called by all 256 threads.
__device__ __forceinline__ void decay_and_tiles(const uint16_t *sq16, const uint16_t *sk16,
                                                const float *sg, const uint32_t *valid,
                                                const PrepTiles &t, float (*part)[kDK],
                                                float *decay, const float *beta_in,
                                                float *beta_out, const ExactRows &xr, int tid) {
  const int cp = tid & 63, qt = tid >> 6, c = 2 * cp;
  const uint32_t vbits = valid[qt >> 1] >> ((qt & 1) * 16);
  float a0[16], a1[16];
  float t0 = 1.f, t1 = 1.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float2 la = *reinterpret_cast<const float2 *>(sg + (qt * 16 + i) * kDK + c);
    if (!((vbits >> i) & 1u)) la = make_float2(0.f, 0.f);
    a0[i] = __expf(la.x);
    a1[i] = __expf(la.y);
    t0 *= a0[i];
    t1 *= a1[i];
  }
  part[qt][c] = t0;
  part[qt][c + 1] = t1;
  if (tid < kC) beta_out[tid] = beta_in[tid];
  if (tid < kDK) xr.tfirst[tid] = kC;
  __syncthreads();
  float pre0 = 1.f, pre1 = 1.f, suf0 = 1.f, suf1 = 1.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float x0 = part[q][c], x1 = part[q][c + 1];
    if (q < qt) { pre0 *= x0; pre1 *= x1; }
    if (q > qt) { suf0 *= x0; suf1 *= x1; }
  }
  const float GC0 = pre0 * t0 * suf0, GC1 = pre1 * t1 * suf1;   // e^{g_C}
  if (qt == 0) {
    decay[c] = GC0;
    decay[c + 1] = GC1;
  }
  bool mk0 = false, mk1 = false;
  const uint32_t *sq = reinterpret_cast<const uint32_t *>(sq16);
  const uint32_t *sk = reinterpret_cast<const uint32_t *>(sk16);
  const int kb = c >> 6, ch = (c & 63) >> 3;
  const uint32_t colq = (uint32_t)(kb * t.qg_R * 128 + (c & 7) * 2);
  const uint32_t colk = (uint32_t)(kb * t.kg_R * 128 + (c & 7) * 2);
  const uint32_t col64 = (uint32_t)(kb * 64 * 128 + (c & 7) * 2);
  // forward: e^{g_r} -> Q G, K G and K e^{-g}
  float e0 = pre0, e1 = pre1;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = qt * 16 + i;                      // r & 7 == i & 7 (row offsets are multiples of 8)
    const uint32_t sw = (uint32_t)((ch ^ (i & 7)) << 4);
    const bool vr = (vbits >> i) & 1u;
    const uint32_t qq = vr ? sq[r * 64 + cp] : 0u, kk = vr ? sk[r * 64 + cp] : 0u;
    const float qa = __uint_as_float(qq << 16), qb = __uint_as_float(qq & 0xFFFF0000u);
    const float ka = __uint_as_float(kk << 16), kb2 = __uint_as_float(kk & 0xFFFF0000u);
    e0 *= a0[i];
    e1 *= a1[i];
    *reinterpret_cast<uint32_t *>(t.qg + colq + (uint32_t)((t.qg_row0 + r) * 128) + sw) =
        pack_bf16x2(qa * e0, qb * e1);
    *reinterpret_cast<uint32_t *>(t.kg + colk + (uint32_t)((t.kg_row0 + r) * 128) + sw) =
        pack_bf16x2(ka * e0, kb2 * e1);
    *reinterpret_cast<uint32_t *>(t.kh + col64 + (uint32_t)(r * 128) + sw) =
        pack_bf16x2(kh_entry(ka, e0, r, c, xr, mk0), kh_entry(kb2, e1, r, c + 1, xr, mk1));
  }
  // backward: e^{g_C - g_r} -> K e^{g_C - g}
  float s0 = suf0, s1 = suf1;
#pragma unroll
  for (int i = 15; i >= 0; --i) {
    const int r = qt * 16 + i;
    const uint32_t sw = (uint32_t)((ch ^ (i & 7)) << 4);
    const bool vr = (vbits >> i) & 1u;
    const uint32_t kk = vr ? sk[r * 64 + cp] : 0u;
    const float ka = __uint_as_float(kk << 16), kb2 = __uint_as_float(kk & 0xFFFF0000u);
    const uint32_t rr = (uint32_t)(r * 128) + sw;
    *reinterpret_cast<uint32_t *>(t.kt + col64 + rr) = pack_bf16x2(ka * s0, kb2 * s1);
    s0 *= a0[i];
    s1 *= a1[i];
  }
}

// P1 reading q, k, log_alpha straight from global memory (rows of the chunk at
// packed positions c0 .. c0+63 of head h; invalid rows count as zero; with a
// head-wise gate log_alpha is [N, H] and every channel takes the row's value).  Besides the
// shared tiles (Q G and K G rows of `t.qg/t.kg`, K e^{-g} in `t.kh`), it writes
// Q G into rows 64.. of the 128-row output tile `gq` (if not null) and K e^{g_C - g}
// into the 64-row tile `gkt` (global or shared memory, same swizzled layout), and
// e^{g_C} into `gdecay` (global) and `decay` (shared).  One __syncthreads(); 256 threads.
// beta_val (threads 0..63: beta of row tid, already in a register) is stored to
// beta_out after the row loads are issued, so its latency overlaps theirs.  With
// `sla` (and `sq`, `sk`), log_alpha (and q, k) come from staged [64][128] row-major
// tiles instead of global memory; they are read before the internal barrier, so the
// operand tiles may be written over them.
template <bool GATE_HEAD>
__device__ __forceinline__ void decay_and_tiles_global(
    const uint16_t *q, const uint16_t *k, const float *log_alpha, int c0, int h, int H,
    const uint32_t *valid, const PrepTiles &t, unsigned char *gq, unsigned char *gkt,
    float *gdecay, float (*part)[kDK], float *decay, float beta_val, float *beta_out,
    const ExactRows &xr, int tid, bool wait_bulk = false, const float *sla = nullptr,
    const uint16_t *sq = nullptr, const uint16_t *sk = nullptr) {
  // thread: channels c .. c+3 (c = 4 (tid % 32)), rows 8 qt .. 8 qt + 7 (qt = tid / 32); 16-byte
  // log_alpha and 8-byte q, k, tile accesses
  const int cq = tid & 31, qt = tid >> 5, c = 4 * cq;
  const uint32_t vbits = (valid[qt >> 2] >> ((qt & 3) * 8)) & 0xFFu;
  float a[8][4];
  uint2 qv[8], kv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool vr = (vbits >> i) & 1u;
    const int rr = qt * 8 + i;
    const size_t row = ((size_t)(c0 + rr) * H + h) * kDK + c;
    float4 la = make_float4(0.f, 0.f, 0.f, 0.f);
    qv[i] = make_uint2(0u, 0u);
    kv[i] = make_uint2(0u, 0u);
    if (vr) {
      if (GATE_HEAD) {
        const float gv = __ldg(log_alpha + (size_t)(c0 + rr) * H + h);
        la = make_float4(gv, gv, gv, gv);
      } else if (sla) {
        la = *reinterpret_cast<const float4 *>(sla + rr * kDK + c);
      } else {
        la = __ldg(reinterpret_cast<const float4 *>(log_alpha + row));
      }
      if (sq) {
        qv[i] = *reinterpret_cast<const uint2 *>(sq + rr * kDK + c);
        kv[i] = *reinterpret_cast<const uint2 *>(sk + rr * kDK + c);
      } else {
        qv[i] = __ldg(reinterpret_cast<const uint2 *>(q + row));
        kv[i] = __ldg(reinterpret_cast<const uint2 *>(k + row));
      }
    }
    a[i][0] = la.x;
    a[i][1] = la.y;
    a[i][2] = la.z;
    a[i][3] = la.w;
  }
  float tt[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[i][e] = __expf(a[i][e]);
      tt[e] *= a[i][e];
    }
  *reinterpret_cast<float4 *>(&part[qt][c]) = make_float4(tt[0], tt[1], tt[2], tt[3]);
  if (tid < kC) beta_out[tid] = beta_val;
  if (tid < kDK) xr.tfirst[tid] = kC;
  // the tiles may still be read by bulk stores thread 0 issued earlier; the tile
  // writes below come after this barrier
  if (wait_bulk && tid == 0) tc::bulk_wait_read();
  __syncthreads();
  float pre[4] = {1.f, 1.f, 1.f, 1.f}, suf[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
  for (int qq = 0; qq < 8; ++qq) {
    const float4 x = *reinterpret_cast<const float4 *>(&part[qq][c]);
    const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (qq < qt) pre[e] *= xv[e];
      if (qq > qt) suf[e] *= xv[e];
    }
  }
  if (qt == 0) {
    const float4 gc = make_float4(pre[0] * tt[0] * suf[0], pre[1] * tt[1] * suf[1], pre[2] * tt[2] * suf[2],
                                  pre[3] * tt[3] * suf[3]);   // e^{g_C}
    *reinterpret_cast<float4 *>(decay + c) = gc;
    if (gdecay) *reinterpret_cast<float4 *>(gdecay + c) = gc;
  }
  bool mk[4] = {false, false, false, false};
  const int kb = c >> 6, ch = (c & 63) >> 3;
  const uint32_t colq = (uint32_t)(kb * t.qg_R * 128 + (c & 7) * 2);
  const uint32_t colk = (uint32_t)(kb * t.kg_R * 128 + (c & 7) * 2);
  const uint32_t col128 = (uint32_t)(kb * 128 * 128 + (c & 7) * 2);
  const uint32_t col64 = (uint32_t)(kb * 64 * 128 + (c & 7) * 2);
  auto unpack = [](uint2 w, float (&x)[4]) {
    x[0] = __uint_as_float(w.x << 16);
    x[1] = __uint_as_float(w.x & 0xFFFF0000u);
    x[2] = __uint_as_float(w.y << 16);
    x[3] = __uint_as_float(w.y & 0xFFFF0000u);
  };
  auto pack4 = [](const float (&x)[4]) { return make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3])); };
  float ev[4] = {pre[0], pre[1], pre[2], pre[3]};
  // e^{g} never increases down the rows (every alpha <= 1), so when this thread's last row
  // is well above the range threshold (the factor 2 covers the rounding of pre * t against
  // the running product), every row passes the range test: it is skipped, same values.
  auto rows = [&](auto fast) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = qt * 8 + i;
      const uint32_t sw = (uint32_t)((ch ^ (r & 7)) << 4);
      float qf[4], kf[4], x[4];
      unpack(qv[i], qf);
      unpack(kv[i], kf);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ev[e] *= a[i][e];
        x[e] = qf[e] * ev[e];
      }
      const uint2 qgv = pack4(x);
      *reinterpret_cast<uint2 *>(t.qg + colq + (uint32_t)((t.qg_row0 + r) * 128) + sw) = qgv;
      if (gq) *reinterpret_cast<uint2 *>(gq + col128 + (uint32_t)((64 + r) * 128) + sw) = qgv;
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = kf[e] * ev[e];
      *reinterpret_cast<uint2 *>(t.kg + colk + (uint32_t)((t.kg_row0 + r) * 128) + sw) = pack4(x);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if constexpr (decltype(fast)::value) {
          float inv;
          asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(ev[e]));
          x[e] = kf[e] * inv;
        } else {
          x[e] = kh_entry(kf[e], ev[e], r, c + e, xr, mk[e]);
        }
      }
      *reinterpret_cast<uint2 *>(t.kh + col64 + (uint32_t)(r * 128) + sw) = pack4(x);
    }
  };
  bool fast = true;
#pragma unroll
  for (int e = 0; e < 4; ++e) fast = fast && (pre[e] * tt[e] > 2.f * kFastMinDecay);
  if (fast)
    rows(BoolTag<true>{});
  else
    rows(BoolTag<false>{});
  float sv[4] = {suf[0], suf[1], suf[2], suf[3]};
#pragma unroll
  for (int i = 7; i >= 0; --i) {
    const int r = qt * 8 + i;
    const uint32_t sw = (uint32_t)((ch ^ (r & 7)) << 4);
    float kf[4], x[4];
    unpack(kv[i], kf);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[e] = kf[e] * sv[e];
      sv[e] *= a[i][e];
    }
    *reinterpret_cast<uint2 *>(gkt + col64 + (uint32_t)(r * 128) + sw) = pack4(x);
  }
}

// 32 fp32 values -> bf16 into 4 consecutive 16-byte chunks (chunk0..chunk0+3) of row r
// of a K-major row tile with R rows and one 64-column block.
__device__ __forceinline__ void store_row32(unsigned char *tile, int R, int r, int chunk0,
                                            const float *v) {
#pragma unroll
  for (int j = 0; j < 32; j += 8) {
    uint4 pk;
    pk.x = pack_bf16x2(v[j + 0], v[j + 1]);
    pk.y = pack_bf16x2(v[j + 2], v[j + 3]);
    pk.z = pack_bf16x2(v[j + 4], v[j + 5]);
    pk.w = pack_bf16x2(v[j + 6], v[j + 7]);
    *reinterpret_cast<uint4 *>(tile + row_tile_chunk(r, 0, chunk0 + (j >> 3), R)) = pk;
  }
}

// P3.  The Gram accumulator (TMEM, 64 columns at `gram_col`) holds M in lanes 0-63
// and A / beta in lanes 64-127.  Writes tril_0(M) as bf16 into rows m_row0.. of the
// 64-column tile `mtile` (R rows) and beta_r * tril_{-1}(A) into As ([64][65] f32).
__device__ __forceinline__ void extract_gram(uint32_t tm_cols, unsigned char *mtile, int mR,
                                             int m_row0, float *As, const float *beta, int tid) {
  const int lr = tid & 127, wg = tid >> 7;
  float v[32];
  tmem_ld32(tm_cols, v);
  if (lr < kC) {
    const int r = lr;
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = (wg * 32 + j <= r) ? v[j] : 0.f;
    store_row32(mtile, mR, m_row0 + r, wg * 4, v);
  } else {
    const int r = lr - kC;
    const float br = beta[r];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int i = wg * 32 + j;
      As[r * 65 + i] = (i < r) ? br * v[j] : 0.f;
    }
  }
}

// T_b = T Diag(beta) (lower part of T in Ts [64][LDT] f32) -> bf16 rows 0..63 of `ttile` (R rows).
// With LDT a multiple of 4 the row is read 16 bytes at a time.
template <int LDT = 65>
__device__ __forceinline__ void pack_tb(const float *Ts, const float *beta, unsigned char *ttile,
                                        int R, int tid) {
  const int r = tid >> 2, qq = tid & 3;      // row r, columns 16qq .. 16qq+15
  float t[16];
  if constexpr (LDT % 4 == 0) {
#pragma unroll
    for (int u = 0; u < 16; u += 4) {
      const float4 x = *reinterpret_cast<const float4 *>(Ts + r * LDT + qq * 16 + u);
      const float4 b = *reinterpret_cast<const float4 *>(beta + qq * 16 + u);
      const float xv[4] = {x.x * b.x, x.y * b.y, x.z * b.z, x.w * b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) t[u + e] = (qq * 16 + u + e <= r) ? xv[e] : 0.f;
    }
  } else {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int i = qq * 16 + u;
      t[u] = (i <= r) ? Ts[r * LDT + i] * beta[i] : 0.f;
    }
  }
#pragma unroll
  for (int j = 0; j < 16; j += 8) {
    uint4 pk;
    pk.x = pack_bf16x2(t[j + 0], t[j + 1]);
    pk.y = pack_bf16x2(t[j + 2], t[j + 3]);
    pk.z = pack_bf16x2(t[j + 4], t[j + 5]);
    pk.w = pack_bf16x2(t[j + 6], t[j + 7]);
    *reinterpret_cast<uint4 *>(ttile + row_tile_chunk(r, 0, (qq * 16 + j) >> 3, R)) = pk;
  }
}

// Exact Gram terms of the exact-path key rows (see the range note at the top).  The
// tensor-core Gram in TMEM (lanes 0-63: M rows, lanes 64-127: rows of K K^T before
// beta; this thread's 32 columns at `tm_acc`) holds every other term; this adds,
// for each channel c with a threshold row t_c and each key row i >= t_c, i <= r,
//   x[r][c] k[i][c] prod_{i < t <= r} alpha[t][c]      (x = q for M rows, k for A rows)
// with running products of alpha (all factors <= 1).  Columns left of every
// threshold are not touched.  Rows outside `valid` count as alpha = 1, q = k = 0
// (identity steps).  q, k and log_alpha are read from global memory (rows c0 ..
// c0 + 63 of head h).  `stage`: >= 12816 bytes of shared memory, free again
// when the function returns.  All 256 threads; contains __syncthreads().  The
// caller skips it when no channel has a threshold row.
template <bool GATE_HEAD>
__device__ __noinline__ void exact_gram_fixup(uint32_t tm_acc, const ExactRows &xr,
                                              const uint32_t *valid, const uint16_t *q,
                                              const uint16_t *k, const float *log_alpha, int c0,
                                              int h, int H, float *stage, int tid) {
  int *list = reinterpret_cast<int *>(stage);   // channels with a threshold row, ascending
  int *tmin = list + kDK;                       // the smallest threshold row
  float *sa = stage + 132;                      // [16][64] alpha of a group of channels
  float *sx = sa + 16 * 64;                     // [16][64] q
  float *sk = sx + 16 * 64;                     // [16][64] k
  const uint32_t *unsafe = xr.unsafe;
  const int n = __popc(unsafe[0]) + __popc(unsafe[1]) + __popc(unsafe[2]) + __popc(unsafe[3]);
  if (tid == 0) *tmin = kC;
  __syncthreads();
  if (tid < kDK) {
    const uint32_t w = unsafe[tid >> 5], bit = 1u << (tid & 31);
    if (w & bit) {
      int pos = __popc(w & (bit - 1u));
      for (int j = 0; j < (tid >> 5); ++j) pos += __popc(unsafe[j]);
      list[pos] = tid;
      atomicMin(tmin, xr.tfirst[tid]);
    }
  }
  const int L = tid & 127, wg = tid >> 7, r = L & 63;
  const bool rowA = L >= kC;
  const int ibase = wg * 32;
  const int ihi = min(ibase + 31, r);
  float acc[32];
#pragma unroll
  for (int u = 0; u < 32; ++u) acc[u] = 0.f;
  for (int g0 = 0; g0 < n; g0 += 16) {
    __syncthreads();   // the list is written; the previous group's reads are done
    for (int e = tid; e < 16 * kC; e += 256) {
      const int j = e >> 6, rr = e & 63;
      float a = 1.f, xq = 0.f, xk = 0.f;
      if (g0 + j < n && ((valid[rr >> 5] >> (rr & 31)) & 1u)) {
        const int c = list[g0 + j];
        const size_t row = (size_t)(c0 + rr) * H + h;
        a = __expf(GATE_HEAD ? log_alpha[row] : log_alpha[row * kDK + c]);
        xq = bf16_to_f32(q[row * kDK + c]);
        xk = bf16_to_f32(k[row * kDK + c]);
      }
      sa[j * kC + rr] = a;
      sx[j * kC + rr] = xq;
      sk[j * kC + rr] = xk;
    }
    __syncthreads();
    const int jn = min(16, n - g0);
    for (int j = 0; j < jn; ++j) {
      const float *aj = sa + j * kC, *kj = sk + j * kC;
      const int tc = xr.tfirst[list[g0 + j]];
      float xP = rowA ? kj[r] : sx[j * kC + r];
      for (int t = ihi + 1; t <= r; ++t) xP *= aj[t];      // prod over (ihi, r]
#pragma unroll
      for (int u = 31; u >= 0; --u) {
        const int i = ibase + u;
        if (i <= r) {
          if (i >= tc) acc[u] = fmaf(xP, kj[i], acc[u]);
          xP *= aj[i];
        }
      }
    }
  }
  const int t0 = *tmin;
  float v[32];
  tmem_ld32(tm_acc, v);
#pragma unroll
  for (int u = 0; u < 32; ++u)
    if (ibase + u >= t0) v[u] += acc[u];
  tmem_st32(tm_acc, v);
  tmem_st_wait();
  __syncthreads();   // every thread is done with `stage` before the caller reuses it
}

__device__ __forceinline__ bool any_unsafe(const uint32_t *unsafe) {
  return (unsafe[0] | unsafe[1] | unsafe[2] | unsafe[3]) != 0u;
}

}  // namespace prep
}  // namespace kda
