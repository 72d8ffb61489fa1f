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
// Every column of the state follows its own recursion given the key-side vectors,
// so the work splits over 16-column d_v slices: u, du, dp, dv and G's columns stay
// in one CTA, while the row sums behind dq, dk, dlog_alpha and dbeta are sums of
// per-slice shares, added into zeroed outputs.  Two kernels, one CTA per
// (sequence, head, slice): the first replays the forward and stores the state
// before every position (workspace [N, H, dk, dv] fp32); the second walks the
// positions backwards, the state it needs prefetched into shared memory with
// cp.async while the current step runs, G resident in shared memory.
// Token-serial fp32: a reference-grade backward, not a tuned one.  Pads are
// identity steps: zero gradients there, G passes through.
#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kSW = 16;          // d_v columns per CTA (each column's recursion is independent)
constexpr int kQ = kSW / 4;      // float4 per row of a slice
constexpr int kCG = 128 / kSW;   // column-sum row groups in the grad kernel (threads 128..255)

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

// One position's vectors, one element per thread (thread t: key channel t and
// column t of the CTA's d_v slice), fetched a step ahead so the global-load
// latency overlaps the current step.
struct Vec {
  float k, q, v, la, dout, beta;
};

template <bool BF16>
__device__ __forceinline__ Vec fetch(const BackwardParams &p, size_t pos, int h, int j0, int tid, bool grad) {
  Vec r = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const size_t bh = pos * p.H + h;
  if (tid < p.dk) {
    r.k = load_elem<BF16>(p.k, bh * p.dk + tid);
    if (grad) r.q = load_elem<BF16>(p.q, bh * p.dk + tid);
    r.la = p.log_alpha[la_index(pos, h, p.H, p.dk, tid, p.gate_head)];
  }
  if (tid < kSW) {
    r.v = load_elem<BF16>(p.v, bh * p.dv + j0 + tid);
    if (grad) r.dout = p.d_o[bh * p.dv + j0 + tid];
  }
  r.beta = p.beta[bh];
  return r;
}

// Forward replay: ws[pos] = the state before position pos (pads included), this
// CTA's kSW columns.  The write k u^T of one position is applied in the same pass
// that stores the next position's state and decays it.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) states_kernel(BackwardParams p) {
  __shared__ __align__(16) float S[128 * kSW];          // [dk][kSW]: decayed, write pending
  __shared__ float kbuf[2][128], sa[128], sv[kSW], su[kSW], part[kThreads / kSW][kSW];
  if (device_error_latched(p.err)) return;
  const int ns = p.dv / kSW, sl = blockIdx.x % ns, bhi = blockIdx.x / ns;
  const int b = bhi / p.H, h = bhi % p.H, tid = threadIdx.x, j0 = sl * kSW;
  const int DK = p.dk, DV = p.dv, n4 = DK * kSW / 4;
  const int cb = p.cu[b], ce = p.cu[b + 1];
  if (cb < 0 || ce < cb || ce > p.N) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_CHECK);
    return;
  }
  float4 *S4 = reinterpret_cast<float4 *>(S);
  const float *I = p.init_state ? p.init_state + ((size_t)b * p.H + h) * DK * DV : nullptr;
  for (int e = tid; e < n4; e += kThreads) {
    const int i = e / kQ, c = (e % kQ) * 4;
    S4[e] = I ? *reinterpret_cast<const float4 *>(I + (size_t)i * DV + j0 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  Vec nxt = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (ce > cb) nxt = fetch<BF16>(p, (size_t)cb, h, j0, tid, false);
  bool pend = false;          // S still lacks the previous position's k u^T (k in kbuf[kp])
  int kp = 0;
  const int cc = tid & (kSW - 1), rg = tid / kSW, rows = DK / (kThreads / kSW);
  for (int pos = cb; pos < ce; ++pos) {
    float *W = p.ws + ((size_t)pos * p.H + h) * DK * DV + j0;
    const bool valid = p.mask == nullptr || p.mask[pos] != 0;
    const Vec cur = nxt;
    if (pos + 1 < ce) nxt = fetch<BF16>(p, (size_t)pos + 1, h, j0, tid, false);
    float *kn = kbuf[kp ^ 1];
    if (tid < DK) {
      kn[tid] = cur.k;
      sa[tid] = valid ? __expf(cur.la) : 1.f;
    }
    if (tid < kSW) sv[tid] = cur.v;
    __syncthreads();
    // finish the previous write, store the state before pos, decay it
    const float *kpv = kbuf[kp];
    for (int e = tid; e < n4; e += kThreads) {
      const int i = e / kQ, c = (e % kQ) * 4;
      float4 x = S4[e];
      if (pend) {
        const float ki = kpv[i];
        x.x = fmaf(ki, su[c], x.x); x.y = fmaf(ki, su[c + 1], x.y);
        x.z = fmaf(ki, su[c + 2], x.z); x.w = fmaf(ki, su[c + 3], x.w);
      }
      *reinterpret_cast<float4 *>(W + (size_t)i * DV + c) = x;
      const float ai = sa[i];
      x.x *= ai; x.y *= ai; x.z *= ai; x.w *= ai;
      S4[e] = x;
    }
    __syncthreads();
    pend = false;
    if (!valid) continue;
    // p = S'^T k over row groups, then u = beta (v - p): the write is left pending
    float acc = 0.f;
    for (int i = rg * rows; i < (rg + 1) * rows; ++i) acc = fmaf(S[i * kSW + cc], kn[i], acc);
    part[rg][cc] = acc;
    __syncthreads();
    if (tid < kSW) {
      float pj = 0.f;
#pragma unroll
      for (int g = 0; g < kThreads / kSW; ++g) pj += part[g][tid];
      su[tid] = cur.beta * (sv[tid] - pj);
    }
    __syncthreads();
    pend = true;
    kp ^= 1;
  }
}

// Reverse walk over this CTA's kSW columns.  Shared memory: two state buffers (the
// state before the current position and, arriving by cp.async, the one before the
// previous position) and G.  Column-local quantities (u, du, dp, dv, G) stay in the
// CTA; the row sums that feed dq, dk, dlog_alpha and dbeta are this slice's share
// and are added into the (zeroed) outputs.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) grad_kernel(BackwardParams p) {
  extern __shared__ __align__(16) float dyn[];          // two state buffers + G, [dk][kSW] each
  __shared__ float sk[128], sq[128], sa[128], sr1[128], sr4[128];
  __shared__ float sv[kSW], sdo[kSW], sp[kSW], su[kSW], sdp[kSW], sc2[kSW];
  __shared__ float partp[kCG][kSW], partc[kCG][kSW];
  __shared__ float red[kThreads / 32];
  if (device_error_latched(p.err)) return;
  const int ns = p.dv / kSW, sl = blockIdx.x % ns, bhi = blockIdx.x / ns;
  const int b = bhi / p.H, h = bhi % p.H, tid = threadIdx.x, j0 = sl * kSW;
  const int H = p.H, DK = p.dk, DV = p.dv, n4 = DK * kSW / 4;
  const int cb = p.cu[b], ce = p.cu[b + 1];
  if (cb < 0 || ce < cb || ce > p.N) {
    if (tid == 0) atomicOr(p.err, ERR_BIT_CHECK);
    return;
  }
  float *Sbuf[2] = {dyn, dyn + DK * kSW};
  float *G = dyn + 2 * DK * kSW;
  float4 *G4 = reinterpret_cast<float4 *>(G);
  const float *F = p.d_final_state ? p.d_final_state + ((size_t)b * H + h) * DK * DV : nullptr;
  for (int e = tid; e < n4; e += kThreads) {
    const int i = e / kQ, c = (e % kQ) * 4;
    G4[e] = F ? *reinterpret_cast<const float4 *>(F + (size_t)i * DV + j0 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  auto prefetch = [&](int pos, float *dst) {
    const float *src = p.ws + ((size_t)pos * H + h) * DK * DV + j0;
    for (int e = tid; e < n4; e += kThreads) {
      const int i = e / kQ, c = (e % kQ) * 4;
      tc::cp_async16(tc::smem_u32(dst + i * kSW + c), src + (size_t)i * DV + c, 16);
    }
    tc::cp_async_commit();
  };
  int cur = 0;
  Vec nxt = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (ce > cb) {
    prefetch(ce - 1, Sbuf[0]);
    nxt = fetch<BF16>(p, (size_t)ce - 1, h, j0, tid, true);
  }
  const int cc = (tid - 128) & (kSW - 1), cg = (tid - 128) / kSW, crows = DK / kCG;
  for (int pos = ce - 1; pos >= cb; --pos) {
    const size_t bh = (size_t)pos * H + h;
    const bool valid = p.mask == nullptr || p.mask[pos] != 0;
    const Vec cv = nxt;
    if (pos > cb) nxt = fetch<BF16>(p, (size_t)pos - 1, h, j0, tid, true);
    if (!valid) {          // identity step: zero gradients (the summed outputs start at 0), G unchanged
      if (tid < kSW) p.gv[bh * DV + j0 + tid] = 0.f;
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
    if (tid < kSW) {
      sv[tid] = cv.v;
      sdo[tid] = cv.dout;
    }
    const float beta = cv.beta;
    tc::cp_async_wait_all();
    __syncthreads();
    const float *S = Sbuf[cur];
    if (pos > cb) prefetch(pos - 1, Sbuf[cur ^ 1]);   // overlaps the step below
    // ---- pass 1: row sums R1 = S dO, R4 = rowsum(G*S) (threads 0..127), column sums
    //      p = S^T (a*k), C2 = G^T k over kCG row groups (threads 128..255)
    if (tid < 128) {
      const int i = tid;
      if (i < DK) {
        float r1 = 0.f, r4 = 0.f;
#pragma unroll 8
        for (int jj = 0; jj < kSW; ++jj) {
          const int c = (jj + i) & (kSW - 1);            // rotated: conflict-free banks
          const float sij = S[i * kSW + c];
          r1 = fmaf(sij, sdo[c], r1);
          r4 = fmaf(G[i * kSW + c], sij, r4);
        }
        sr1[i] = r1;
        sr4[i] = r4;
      }
    } else {
      float pj = 0.f, c2 = 0.f;
      for (int i = cg * crows; i < (cg + 1) * crows; ++i) {
        pj = fmaf(S[i * kSW + cc], sa[i] * sk[i], pj);
        c2 = fmaf(G[i * kSW + cc], sk[i], c2);
      }
      partp[cg][cc] = pj;
      partc[cg][cc] = c2;
    }
    __syncthreads();
    if (tid < kSW) {
      float pj = 0.f, c2 = 0.f;
#pragma unroll
      for (int g = 0; g < kCG; ++g) {
        pj += partp[g][tid];
        c2 += partc[g][tid];
      }
      sp[tid] = pj;
      sc2[tid] = c2;
      su[tid] = beta * (sv[tid] - pj);
    }
    __syncthreads();
    // ---- q.k (whole key) and this slice's u.dO
    const float qk = block_sum(tid < DK ? sq[tid] * sk[tid] : 0.f, red);
    const float udo = block_sum(tid < kSW ? su[tid] * sdo[tid] : 0.f, red);
    // ---- du, dv, dp; this slice's share of dbeta = du . (v - p)
    float x3 = 0.f;
    if (tid < kSW) {
      const float du = sc2[tid] + qk * sdo[tid];
      p.gv[bh * DV + j0 + tid] = beta * du;
      sdp[tid] = -beta * du;
      x3 = du * (sv[tid] - sp[tid]);
    }
    const float db = block_sum(x3, red);      // its barriers also publish sdp
    if (tid == 0) atomicAdd(p.gbeta + bh, db);
    // ---- pass 2: R2 = G u, R3 = S dp over this slice; shares of dq, dk, dlog_alpha
    float xla = 0.f;
    if (tid < DK) {
      const int i = tid;
      float r2 = 0.f, r3 = 0.f;
#pragma unroll 8
      for (int jj = 0; jj < kSW; ++jj) {
        const int c = (jj + i) & (kSW - 1);
        r2 = fmaf(G[i * kSW + c], su[c], r2);
        r3 = fmaf(S[i * kSW + c], sdp[c], r3);
      }
      const float ai = sa[i];
      atomicAdd(p.gq + bh * DK + i, ai * sr1[i] + sk[i] * udo);
      atomicAdd(p.gk + bh * DK + i, r2 + sq[i] * udo + ai * r3);
      const float dla = ai * (sr4[i] + sq[i] * sr1[i] + sk[i] * r3);
      if (p.gate_head) xla = dla;
      else atomicAdd(p.gla + bh * DK + i, dla);
    }
    if (p.gate_head) {
      const float t = block_sum(xla, red);
      if (tid == 0) atomicAdd(p.gla + bh, t);
    }
    __syncthreads();      // G is read above and rewritten below
    // ---- pass 3: G <- Diag(a) (G + q dO^T + k dp^T)
    for (int e = tid; e < n4; e += kThreads) {
      const int i = e / kQ, c = (e % kQ) * 4;
      const float ai = sa[i], qi = sq[i], ki = sk[i];
      float4 gx = G4[e];
      gx.x = ai * (gx.x + qi * sdo[c] + ki * sdp[c]);
      gx.y = ai * (gx.y + qi * sdo[c + 1] + ki * sdp[c + 1]);
      gx.z = ai * (gx.z + qi * sdo[c + 2] + ki * sdp[c + 2]);
      gx.w = ai * (gx.w + qi * sdo[c + 3] + ki * sdp[c + 3]);
      G4[e] = gx;
    }
    __syncthreads();
    cur ^= 1;
  }
  tc::cp_async_wait_all();
  if (p.g_init_state) {
    float *O = p.g_init_state + ((size_t)b * H + h) * DK * DV + j0;
    for (int e = tid; e < n4; e += kThreads) {
      const int i = e / kQ, c = (e % kQ) * 4;
      *reinterpret_cast<float4 *>(O + (size_t)i * DV + c) = G4[e];
    }
  }
}

}  // namespace bwd

size_t backward_workspace(int N, int H, int dk, int dv) { return (size_t)N * H * dk * dv * 4; }

cudaError_t launch_backward(const BackwardParams &p, bool bf16, cudaStream_t s) {
  using namespace bwd;
  if (p.num_seqs == 0) return cudaSuccess;
  // dq, dk, dlog_alpha and dbeta are sums over the d_v slices
  const size_t nh = (size_t)p.N * p.H;
  cudaError_t e;
  if ((e = cudaMemsetAsync(p.gq, 0, nh * p.dk * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.gk, 0, nh * p.dk * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.gla, 0, nh * (p.gate_head ? 1 : p.dk) * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.gbeta, 0, nh * 4, s)) != cudaSuccess) return e;
  const unsigned grid = (unsigned)p.num_seqs * p.H * (p.dv / kSW);
  if (bf16) states_kernel<true><<<grid, kThreads, 0, s>>>(p);
  else states_kernel<false><<<grid, kThreads, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int gsm = 3 * p.dk * kSW * 4;
  auto kg = bf16 ? grad_kernel<true> : grad_kernel<false>;
  if ((e = cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize, gsm)) != cudaSuccess) return e;
  kg<<<grid, kThreads, gsm, s>>>(p);
  return cudaGetLastError();
}

}  // namespace kda
