// 64 x 64 unit-lower-triangular inverse T = (I + A)^{-1} for the WY/UT form
// of a KDA chunk (the triangular solve that turns a chunk's rank-1 updates into
// dense products; "Kimi Linear's 75% KV cache cut ...", theclarity.today,
// fourth paragraph).
//
// Built from 16 x 16 blocks (the inverse of a block unit-lower-triangular
// matrix [[L11, 0], [L21, L22]] is [[L11^-1, 0], [-L22^-1 L21 L11^-1, L22^-1]]),
// with the 16 x 16 x 16 block products on the tensor cores (warp-level mma.sync
// m16n8k8, TF32 inputs rounded to nearest, fp32 accumulation).  The inverse
// only feeds bf16 operands, so TF32 inputs (2^-11) are below the final
// rounding (2^-9).
//
// Shared arrays are fp32, row-major with stride 65.  A must be strictly lower
// (zeros on and above the diagonal).  Only entries on or below the diagonal of
// T are written with meaningful values; the blocks above the diagonal are not
// touched.
#pragma once

#include <stdint.h>

namespace kda {
namespace tri {

constexpr int kLD = 65;     // default row stride of the [64][.] f32 tiles

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// acc[n] (two 16x8 tiles, n = 0, 1) += X[16 x 16] * Y[16 x 16]; X, Y row-major with stride ldx/ldy.
// Fragment layout of m16n8k8 (g = lane / 4, t = lane % 4):
//   A: a0 = X[g][t], a1 = X[g+8][t], a2 = X[g][t+4], a3 = X[g+8][t+4]
//   B: b0 = Y[t][g], b1 = Y[t+4][g]
//   C: c0 = C[g][2t], c1 = C[g][2t+1], c2 = C[g+8][2t], c3 = C[g+8][2t+1]
__device__ __forceinline__ void block_mma(float (&acc)[2][4], const float *X, int ldx, const float *Y,
                                          int ldy, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int kk = 0; kk < 16; kk += 8) {
    uint32_t a[4];
    a[0] = to_tf32(X[g * ldx + kk + t]);
    a[1] = to_tf32(X[(g + 8) * ldx + kk + t]);
    a[2] = to_tf32(X[g * ldx + kk + t + 4]);
    a[3] = to_tf32(X[(g + 8) * ldx + kk + t + 4]);
#pragma unroll
    for (int n = 0; n < 2; ++n) {
      uint32_t b[2];
      b[0] = to_tf32(Y[(kk + t) * ldy + n * 8 + g]);
      b[1] = to_tf32(Y[(kk + t + 4) * ldy + n * 8 + g]);
      mma_tf32(acc[n], a, b);
    }
  }
}

__device__ __forceinline__ void store_acc(float *Z, int ldz, const float (&acc)[2][4], float scale,
                                          int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    Z[g * ldz + n * 8 + 2 * t] = scale * acc[n][0];
    Z[g * ldz + n * 8 + 2 * t + 1] = scale * acc[n][1];
    Z[(g + 8) * ldz + n * 8 + 2 * t] = scale * acc[n][2];
    Z[(g + 8) * ldz + n * 8 + 2 * t + 1] = scale * acc[n][3];
  }
}

// Scratch: 32 x 33 floats.  Must be called by all 256 threads.
// Recursive doubling: the four 16 x 16 diagonal inverses D_a (registers, one
// thread per column); then the two 32 x 32 diagonal inverses
//   P0 = [[D0, 0], [-D1 A10 D0, D1]],  P1 = [[D2, 0], [-D3 A32 D2, D3]];
// then the lower-left 32 x 32 block -P1 (A_LL P0), with one warp per 16 x 16
// output tile.  The block products are tensor-core MMAs.
template <int LD = kLD>      // row stride of As and Ts (floats)
__device__ __forceinline__ void unit_lower_inverse_64(const float *__restrict__ As,
                                                      float *__restrict__ Ts,
                                                      float *__restrict__ scratch, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  // ---- 16 x 16 diagonal blocks: thread (blk, j) holds column j of D_blk in registers.
  // Right-looking: once t[i] is known it is folded into every later row.
  if (tid < 64) {
    const int blk = tid >> 4, j = tid & 15, o = blk * 16;
    float acc[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) acc[r] = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float ti = (i < j) ? 0.f : (i == j ? 1.f : -acc[i]);
      Ts[(o + i) * LD + o + j] = ti;
#pragma unroll
      for (int r = i + 1; r < 16; ++r) acc[r] = fmaf(As[(o + r) * LD + o + i], ti, acc[r]);
    }
  }
  __syncthreads();
  // ---- 32 x 32 diagonal blocks: warp 0 -> T10 = -D1 A10 D0, warp 1 -> T32 = -D3 A32 D2
  if (warp < 2) {
    const int a = 2 * warp + 1, b = 2 * warp;      // (1,0) or (3,2)
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    block_mma(acc, As + (a * 16) * LD + b * 16, LD, Ts + (b * 16) * LD + b * 16, LD, lane);
    float *X = scratch + warp * 16 * 17;
    store_acc(X, 17, acc, 1.f, lane);
    __syncwarp();
    float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    block_mma(acc2, Ts + (a * 16) * LD + a * 16, LD, X, 17, lane);
    store_acc(Ts + (a * 16) * LD + b * 16, LD, acc2, -1.f, lane);
  }
  __syncthreads();
  // ---- lower-left 32 x 32: X = A[32:64, 0:32] P0 (tile (i, j) sums m = j..1), one warp per tile
  float *X = scratch;                             // 32 x 33
  if (warp < 4) {
    const int i = warp >> 1, j = warp & 1;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int m = j; m < 2; ++m)
      block_mma(acc, As + (32 + i * 16) * LD + m * 16, LD, Ts + (m * 16) * LD + j * 16, LD, lane);
    store_acc(X + (i * 16) * 33 + j * 16, 33, acc, 1.f, lane);
  }
  __syncthreads();
  // ---- T[32:64, 0:32] = -P1 X (tile (i, j) sums m = 0..i)
  if (warp < 4) {
    const int i = warp >> 1, j = warp & 1;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int m = 0; m <= i; ++m)
      block_mma(acc, Ts + (32 + i * 16) * LD + 32 + m * 16, LD, X + (m * 16) * 33 + j * 16, 33, lane);
    store_acc(Ts + (32 + i * 16) * LD + j * 16, LD, acc, -1.f, lane);
  }
  __syncthreads();
}

}  // namespace tri
}  // namespace kda
