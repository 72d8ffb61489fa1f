// Backward pass of the KDA prefill: gradients of <o, dO> + <S_final, dS_final> with
// respect to q, k, v, log_alpha, beta and the initial state.
//
// The forward step at a valid position (the operator's definition: "Kimi Linear's
// 75% KV cache cut ...", theclarity.today, third paragraph; the delta rule of
// "Kimi Linear wlasnie pokonal ...", remio.ai, section "Jak Kimi Linear
// wykorzystuje inteligentniejsza pamiec rekurencyjna"):
//   S' = Diag(a) S,  a = exp(log_alpha);  p = S'^T k;  u = beta (v - p);
//   S  = S' + k u^T;  o = S^T q.
// Reverse mode, with G the gradient of the state after the step:
//   G += q dO^T;  dq = S dO;  dk = G u + S' dp;  du = G^T k;  dv = beta du;
//   dbeta = du . (v - p);  dp = -beta du;  dlog_alpha = rowsum((G + k dp^T) * S');
//   G <- Diag(a) (G + k dp^T).
// Expanded so that no intermediate matrix is materialised: with
//   R1 = S dO, R2 = G u, R3 = S dp, R4 = rowsum(G * S)  (row sums of the stored S)
//   p = S^T (a*k), C2 = G^T k                            (column sums)
// one gets dq = a*R1 + k (u.dO), dk = R2 + q (dO.u) + a*R3,
// du = C2 + (q.k) dO and dlog_alpha = a * (R4 + q*R1 + k*R3).
//
// Two kernels, one CTA per (sequence, head): the first replays the forward and
// stores the state before every position (workspace [N, H, dk, dv] fp32); the
// second walks the positions backwards, the state it needs prefetched into
// shared memory with cp.async while the current step runs, G resident in shared
// memory.  Token-serial fp32: a reference-grade backward, not a tuned one.  Pads
// are identity steps: zero gradients there, G passes through.
#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace bwd {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_sum(float x, float *red) {
  // sum over the CTA's 256 threads (every thread gets the result)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = x;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < kThreads / 32; ++i) t += red[i];
  return t;
}

// One position's vectors, one element per thread (thread t: key channel t, value
// column t; head dims are at most 128 < 256 threads), fetched a step ahead so the
// global-load latency overlaps the current step.
struct Vec {
  float k, q, v, la, dout, beta;
};

template <bool BF16>
__device__ __forceinline__ Vec fetch(const BackwardParams &p, size_t pos, int h, int tid, bool grad) {
  Vec r = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const size_t bh = pos * p.H + h;
  if (tid < p.dk) {
    r.k = load_elem<BF16>(p.k, bh * p.dk + tid);
    if (grad) r.q = load_elem<BF16>(p.q, bh * p.dk + tid);
    r.la = p.log_alpha[la_index(pos, h, p.H, p.dk, tid, p.gate_head)];
  }
  if (tid < p.dv) {
    r.v = load_elem<BF16>(p.v, bh * p.dv + tid);
    if (grad) r.dout = p.d_o[bh * p.dv + tid];
  }
  r.beta = p.beta[bh];
  return r;
}

// Forward replay: ws[pos] = the state before position pos (pads included).  The
// write k u^T of one position is applied in the same pass that stores the next
// position's state and decays it, so each position costs one elementwise pass.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) states_kernel(BackwardParams p) {
  extern __shared__ __align__(16) float S[];            // [dk][dv]: decayed, write pending
  __shared__ float kbuf[2][128], sv[128], sa[128], su[128];
  if (device_error_latched(p.err)) return;
  const int b = blockIdx.x / p.H, h = blockIdx.x % p.H, tid = threadIdx.x;
  const int DK = p.dk, DV = p.dv, n4 = DK * DV / 4;
  const int dv_shift = 31 - __clz(DV);                  // head dims are powers of two
  const int cb = p.cu[b], ce = p.cu[b + 1];
  if (cb < 0 || ce < cb || ce > p.N) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_CHECK);
    return;
  }
  float4 *S4 = reinterpret_cast<float4 *>(S);
  const float4 *I4 = p.init_state ? reinterpret_cast<const float4 *>(p.init_state + ((size_t)b * p.H + h) * DK * DV)
                                  : nullptr;
  for (int e = tid; e < n4; e += kThreads) S4[e] = I4 ? I4[e] : make_float4(0.f, 0.f, 0.f, 0.f);
  Vec nxt = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (ce > cb) nxt = fetch<BF16>(p, (size_t)cb, h, tid, false);
  bool pend = false;          // S still lacks the previous position's k u^T (k in kbuf[kp])
  int kp = 0;
  for (int pos = cb; pos < ce; ++pos) {
    float4 *W4 = reinterpret_cast<float4 *>(p.ws + ((size_t)pos * p.H + h) * DK * DV);
    const bool valid = p.mask == nullptr || p.mask[pos] != 0;
    const Vec cur = nxt;
    if (pos + 1 < ce) nxt = fetch<BF16>(p, (size_t)pos + 1, h, tid, false);
    float *kn = kbuf[kp ^ 1];
    if (tid < DK) {
      kn[tid] = cur.k;
      sa[tid] = valid ? __expf(cur.la) : 1.f;
    }
    if (tid < DV) sv[tid] = cur.v;
    __syncthreads();
    // finish the previous write, store the state before pos, decay it
    const float *kpv = kbuf[kp];
    for (int e = tid; e < n4; e += kThreads) {
      const int i = (4 * e) >> dv_shift, j = (4 * e) & (DV - 1);
      float4 x = S4[e];
      if (pend) {
        const float ki = kpv[i];
        x.x = fmaf(ki, su[j], x.x); x.y = fmaf(ki, su[j + 1], x.y);
        x.z = fmaf(ki, su[j + 2], x.z); x.w = fmaf(ki, su[j + 3], x.w);
      }
      W4[e] = x;
      const float ai = sa[i];
      x.x *= ai; x.y *= ai; x.z *= ai; x.w *= ai;
      S4[e] = x;
    }
    __syncthreads();
    pend = false;
    if (!valid) continue;
    // p = S'^T k, u = beta (v - p): the write of this position is left pending
    for (int j = tid; j < DV; j += kThreads) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int i = 0; i < DK; i += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u] = fmaf(S[(i + u) * DV + j], kn[i + u], acc[u]);
      }
      su[j] = cur.beta * (sv[j] - ((acc[0] + acc[1]) + (acc[2] + acc[3])));
    }
    __syncthreads();
    pend = true;
    kp ^= 1;
  }
}

// Reverse walk.  Shared memory: two state buffers (the state before the current
// position and, arriving by cp.async, the one before the previous position) and G.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) grad_kernel(BackwardParams p) {
  extern __shared__ __align__(16) float smem[];
  __shared__ float sk[128], sq[128], sv[128], sa[128], sdo[128];
  __shared__ float sp[128], su[128], sdp[128], sc2[128], sr1[128], sr4[128];
  __shared__ float sr2[2][128], sr3[2][128];
  __shared__ float red[kThreads / 32];
  if (device_error_latched(p.err)) return;
  const int b = blockIdx.x / p.H, h = blockIdx.x % p.H, tid = threadIdx.x;
  const int H = p.H, DK = p.dk, DV = p.dv, n4 = DK * DV / 4, MS = DK * DV;
  const int dv_shift = 31 - __clz(DV);                  // head dims are powers of two
  const int cb = p.cu[b], ce = p.cu[b + 1];
  if (cb < 0 || ce < cb || ce > p.N) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_CHECK);
    return;
  }
  float *Sbuf[2] = {smem, smem + MS};
  float *G = smem + 2 * MS;
  float4 *G4 = reinterpret_cast<float4 *>(G);
  const float4 *F4 = p.d_final_state ? reinterpret_cast<const float4 *>(p.d_final_state + ((size_t)b * H + h) * MS)
                                     : nullptr;
  for (int e = tid; e < n4; e += kThreads) G4[e] = F4 ? F4[e] : make_float4(0.f, 0.f, 0.f, 0.f);
  auto prefetch = [&](int pos, float *dst) {
    const float *src = p.ws + ((size_t)pos * H + h) * MS;
    for (int e = tid; e < n4; e += kThreads)
      tc::cp_async16(tc::smem_u32(dst + 4 * e), src + 4 * e, 16);
    tc::cp_async_commit();
  };
  int cur = 0;
  Vec nxt = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (ce > cb) {
    prefetch(ce - 1, Sbuf[0]);
    nxt = fetch<BF16>(p, (size_t)ce - 1, h, tid, true);
  }
  for (int pos = ce - 1; pos >= cb; --pos) {
    const size_t bh = (size_t)pos * H + h;
    const bool valid = p.mask == nullptr || p.mask[pos] != 0;
    const Vec cv = nxt;
    if (pos > cb) nxt = fetch<BF16>(p, (size_t)pos - 1, h, tid, true);
    if (!valid) {          // identity step: zero gradients, G unchanged
      for (int c = tid; c < DK; c += kThreads) {
        p.gq[bh * DK + c] = 0.f;
        p.gk[bh * DK + c] = 0.f;
        if (!p.gate_head) p.gla[bh * DK + c] = 0.f;
      }
      for (int j = tid; j < DV; j += kThreads) p.gv[bh * DV + j] = 0.f;
      if (tid == 0) {
        p.gbeta[bh] = 0.f;
        if (p.gate_head) p.gla[bh] = 0.f;
      }
      tc::cp_async_wait_all();
      __syncthreads();
      if (pos > cb) prefetch(pos - 1, Sbuf[cur]);     // the same buffer: this one was not used
      continue;
    }
    if (tid < DK) {
      sk[tid] = cv.k;
      sq[tid] = cv.q;
      sa[tid] = __expf(cv.la);
    }
    if (tid < DV) {
      sv[tid] = cv.v;
      sdo[tid] = cv.dout;
    }
    const float beta = cv.beta;
    tc::cp_async_wait_all();
    __syncthreads();
    const float *S = Sbuf[cur];
    if (pos > cb) prefetch(pos - 1, Sbuf[cur ^ 1]);   // overlaps the step below
    // ---- pass 1: column sums (threads 0..127) and row sums (threads 128..255)
    if (tid < 128) {
      for (int j = tid; j < DV; j += 128) {
        float pj[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int i = 0; i < DK; i += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            pj[u] = fmaf(S[(i + u) * DV + j], sa[i + u] * sk[i + u], pj[u]);
            c2[u] = fmaf(G[(i + u) * DV + j], sk[i + u], c2[u]);
          }
        }
        sp[j] = (pj[0] + pj[1]) + (pj[2] + pj[3]);
        sc2[j] = (c2[0] + c2[1]) + (c2[2] + c2[3]);
      }
    } else {
      for (int i = tid - 128; i < DK; i += 128) {
        float r1[4] = {0.f, 0.f, 0.f, 0.f}, r4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int jj = 0; jj < DV; jj += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = (i + jj + u) & (DV - 1);          // rotated: conflict-free banks
            const float sij = S[i * DV + j];
            r1[u] = fmaf(sij, sdo[j], r1[u]);
            r4[u] = fmaf(G[i * DV + j], sij, r4[u]);
          }
        }
        sr1[i] = (r1[0] + r1[1]) + (r1[2] + r1[3]);
        sr4[i] = (r4[0] + r4[1]) + (r4[2] + r4[3]);
      }
    }
    __syncthreads();
    for (int j = tid; j < DV; j += kThreads) su[j] = beta * (sv[j] - sp[j]);
    __syncthreads();
    // ---- scalars q.k and u.dO
    float x1 = 0.f, x2 = 0.f;
    for (int c = tid; c < DK; c += kThreads) x1 += sq[c] * sk[c];
    for (int j = tid; j < DV; j += kThreads) x2 += su[j] * sdo[j];
    const float qk = block_sum(x1, red);
    const float udo = block_sum(x2, red);
    // ---- du, dv, dp; dbeta = du . (v - p)
    float x3 = 0.f;
    for (int j = tid; j < DV; j += kThreads) {
      const float du = sc2[j] + qk * sdo[j];
      p.gv[bh * DV + j] = beta * du;
      sdp[j] = -beta * du;
      x3 += du * (sv[j] - sp[j]);
    }
    const float db = block_sum(x3, red);      // its barriers also publish sdp
    if (tid == 0) p.gbeta[bh] = db;
    // ---- pass 2: R2 = G u, R3 = S dp (rows; two threads per row, half the columns each)
    {
      const int i = tid & 127, half = tid >> 7, w = DV / 2;
      if (i < DK) {
        float r2v[4] = {0.f, 0.f, 0.f, 0.f}, r3v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int jj = 0; jj < w; jj += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = (i + half * w + jj + u) & (DV - 1);   // rotated: conflict-free banks
            r2v[u] = fmaf(G[i * DV + j], su[j], r2v[u]);
            r3v[u] = fmaf(S[i * DV + j], sdp[j], r3v[u]);
          }
        }
        sr2[half][i] = (r2v[0] + r2v[1]) + (r2v[2] + r2v[3]);
        sr3[half][i] = (r3v[0] + r3v[1]) + (r3v[2] + r3v[3]);
      }
    }
    __syncthreads();
    // ---- dq, dk, dlog_alpha
    float xla = 0.f;
    for (int i = tid; i < DK; i += kThreads) {
      const float r2 = sr2[0][i] + sr2[1][i], r3 = sr3[0][i] + sr3[1][i];
      const float ai = sa[i];
      p.gq[bh * DK + i] = ai * sr1[i] + sk[i] * udo;
      p.gk[bh * DK + i] = r2 + sq[i] * udo + ai * r3;
      const float dla = ai * (sr4[i] + sq[i] * sr1[i] + sk[i] * r3);
      if (p.gate_head) xla += dla;
      else p.gla[bh * DK + i] = dla;
    }
    if (p.gate_head) {
      const float t = block_sum(xla, red);
      if (tid == 0) p.gla[bh] = t;
    }
    __syncthreads();      // G is read above and rewritten below
    // ---- pass 3: G <- Diag(a) (G + q dO^T + k dp^T)
    for (int e = tid; e < n4; e += kThreads) {
      const int i = (4 * e) >> dv_shift, j = (4 * e) & (DV - 1);
      const float ai = sa[i], qi = sq[i], ki = sk[i];
      float4 gx = G4[e];
      gx.x = ai * (gx.x + qi * sdo[j] + ki * sdp[j]);
      gx.y = ai * (gx.y + qi * sdo[j + 1] + ki * sdp[j + 1]);
      gx.z = ai * (gx.z + qi * sdo[j + 2] + ki * sdp[j + 2]);
      gx.w = ai * (gx.w + qi * sdo[j + 3] + ki * sdp[j + 3]);
      G4[e] = gx;
    }
    __syncthreads();
    cur ^= 1;
  }
  tc::cp_async_wait_all();
  if (p.g_init_state) {
    float4 *O4 = reinterpret_cast<float4 *>(p.g_init_state + ((size_t)b * H + h) * MS);
    for (int e = tid; e < n4; e += kThreads) O4[e] = G4[e];
  }
}

}  // namespace bwd

size_t backward_workspace(int N, int H, int dk, int dv) { return (size_t)N * H * dk * dv * 4; }

cudaError_t launch_backward(const BackwardParams &p, bool bf16, cudaStream_t s) {
  using namespace bwd;
  if (p.num_seqs == 0) return cudaSuccess;
  const unsigned grid = (unsigned)p.num_seqs * p.H;
  const int ms = p.dk * p.dv * 4;
  auto ks = bf16 ? states_kernel<true> : states_kernel<false>;
  auto kg = bf16 ? grad_kernel<true> : grad_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, ms);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize, 3 * ms);
  if (e != cudaSuccess) return e;
  ks<<<grid, kThreads, ms, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kg<<<grid, kThreads, 3 * ms, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
