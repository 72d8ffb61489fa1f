// 64 x 64 unit-lower-triangular inverse T = (I + A)^{-1} for the WY/UT form
// of a KDA chunk (the triangular solve that turns a chunk's rank-1 updates into
// dense products; "Kimi Linear's 75% KV cache cut ...", theclarity.today,
// fourth paragraph).
//
// Blocked by 16: the four diagonal blocks D_a = (I + A_aa)^{-1} by forward
// substitution in registers (one thread per column), then the off-diagonal
// blocks in order of distance d = a - b:
//   T_ab = -D_a * sum_{m=b}^{a-1} A_am T_mb
// with the 16 x 16 x 16 block products on the tensor cores (warp-level
// mma.sync m16n8k8, TF32 inputs rounded to nearest, fp32 accumulation).  The
// inverse only feeds bf16 operands, so TF32 inputs (2^-11) are below the
// final rounding (2^-9).
//
// Shared arrays are fp32, row-major with stride 65.  A must be strictly lower
// (zeros on and above the diagonal).  Only entries on or below the diagonal of
// T are written with meaningful values; the blocks above the diagonal are not
// touched.  Needs 256 threads (8 warps) and a 16 x 17 fp32 scratch per warp.
#pragma once

#include <stdint.h>

namespace kda {
namespace tri {

constexpr int LD = 65;

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

// scratch: 8 warps x 16 x 17 floats.  Must be called by all 256 threads.
__device__ __forceinline__ void unit_lower_inverse_64(const float *__restrict__ As,
                                                      float *__restrict__ Ts,
                                                      float *__restrict__ scratch, int tid) {
  const int warp = tid >> 5, lane = tid & 31;
  // ---- diagonal blocks: thread (blk, j) holds column j of D_blk in registers.
  // Right-looking: once t[i] is known it is folded into every later row, so
  // the dependency depth is 16 steps rather than 120 sequential FMAs.
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
  // ---- off-diagonal blocks by distance
#pragma unroll 1
  for (int d = 1; d <= 3; ++d) {
    if (warp < 4 - d) {
      const int b = warp, a = warp + d;
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      for (int m = b; m < a; ++m)
        block_mma(acc, As + (a * 16) * LD + m * 16, LD, Ts + (m * 16) * LD + b * 16, LD, lane);
      float *X = scratch + warp * 16 * 17;
      store_acc(X, 17, acc, 1.f, lane);
      __syncwarp();
      float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      block_mma(acc2, Ts + (a * 16) * LD + a * 16, LD, X, 17, lane);
      store_acc(Ts + (a * 16) * LD + b * 16, LD, acc2, -1.f, lane);
    }
    __syncthreads();
  }
}

}  // namespace tri
}  // namespace kda
