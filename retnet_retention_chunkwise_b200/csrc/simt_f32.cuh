// simt_f32.cuh -- fp32 CUDA-core kernels for the parallel and chunkwise forms.
//
// fp32 inputs ask for fp32 accuracy end to end.  The tensor cores' fp32-input
// mode (tf32) keeps only 10 explicit mantissa bits per operand, so these forms
// run on FFMA instead: plain tiled kernels with fp32 accumulation.  They serve
// small heads and accuracy-critical callers; the bf16 tensor-core kernels are
// the throughput path.
//
// Decay factors gamma^n (n >= 0) are exp2(n * log2(gamma)) with gamma^0 = 1
// (also for gamma = 0, where log2(gamma) = -inf).
#pragma once
#include <stdint.h>

namespace ret {

struct HeadLog2 {
  float l2g[1024];  // per-head log2(gamma) (RET_MAX_HEADS); -inf for gamma = 0
};

__device__ __forceinline__ float decay_pow(float log2g, int n) {
  return n == 0 ? 1.f : exp2f((float)n * log2g);
}

// ----------------------------------------------------------- parallel form
// y[n] = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m  (page "Retentive Networks --
// Microsoft ...", section "Il meccanismo", parallel form).
// CTA = (64-column block of y, 32 query rows, (b,h)).  Thread (r, cg):
// r = tid / 8 owns query row r, cg = tid % 8 owns columns cg, cg+8, ..., cg+56.
// REV: the anti-causal sum y_n = sum_{m>=n} gamma^(m-n) (q_n . k_m) v_m (key
// tiles from the query tile to the end).
constexpr int kPF_Rows = 32;
constexpr int kPF_Cols = 64;

template <bool REV>
__global__ void __launch_bounds__(256)
parallel_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                    const float* __restrict__ v, float* __restrict__ y, int H, int L, int dk,
                    int dv, const __grid_constant__ HeadLog2 hl) {
  extern __shared__ float sm[];
  const int ldq = dk + 1;
  float* Qs = sm;                          // [32][dk+1]
  float* Ks = Qs + kPF_Rows * ldq;         // [32][dk+1]
  float* Vs = Ks + kPF_Rows * ldq;         // [32][64]
  float* Ps = Vs + kPF_Rows * kPF_Cols;    // [32][33]

  const int bh = blockIdx.z;
  const float l2g = hl.l2g[bh % H];
  const int q0 = blockIdx.y * kPF_Rows, c0 = blockIdx.x * kPF_Cols;
  const int tid = threadIdx.x, r = tid >> 3, cg = tid & 7;
  const float* qh = q + (size_t)bh * L * dk;
  const float* kh = k + (size_t)bh * L * dk;
  const float* vh = v + (size_t)bh * L * dv;

  for (int e = tid; e < kPF_Rows * dk; e += 256) {
    const int i = e / dk, d = e % dk;
    Qs[i * ldq + d] = (q0 + i < L) ? qh[(size_t)(q0 + i) * dk + d] : 0.f;
  }
  float acc[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) acc[u] = 0.f;

  for (int k0 = REV ? q0 : 0; REV ? k0 < L : (k0 <= q0 && k0 < L); k0 += kPF_Rows) {
    __syncthreads();
    for (int e = tid; e < kPF_Rows * dk; e += 256) {
      const int j = e / dk, d = e % dk;
      Ks[j * ldq + d] = (k0 + j < L) ? kh[(size_t)(k0 + j) * dk + d] : 0.f;
    }
    for (int e = tid; e < kPF_Rows * kPF_Cols; e += 256) {
      const int j = e / kPF_Cols, c = e % kPF_Cols;
      Vs[e] = (k0 + j < L && c0 + c < dv) ? vh[(size_t)(k0 + j) * dv + c0 + c] : 0.f;
    }
    __syncthreads();
    // scores for (r, 4 keys), decayed and masked
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = cg * 4 + u;
      float s = 0.f;
      for (int d = 0; d < dk; ++d) s = fmaf(Qs[r * ldq + d], Ks[j * ldq + d], s);
      const int n = REV ? (k0 + j) - (q0 + r) : (q0 + r) - (k0 + j);
      Ps[r * 33 + j] = (n >= 0 && k0 + j < L) ? s * decay_pow(l2g, n) : 0.f;
    }
    __syncthreads();
    for (int j = 0; j < kPF_Rows; ++j) {
      const float p = Ps[r * 33 + j];
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u] = fmaf(p, Vs[j * kPF_Cols + cg + 8 * u], acc[u]);
    }
  }
  if (q0 + r < L) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + cg + 8 * u;
      if (c < dv) y[((size_t)bh * L + q0 + r) * dv + c] = acc[u];
    }
  }
}

// ---------------------------------------------------------- chunkwise form
// Blocks of length C <= 128 (page "Retentive Networks -- Microsoft ...",
// section "Il meccanismo", chunkwise form).  For a block at t0 of length l:
//   y_{t0+i} = sum_{j<=i} gamma^(i-j) (q_i.k_j) v_j + gamma^(i+1) q_i S
//   S       <- gamma^l S + sum_{j<l} gamma^(l-1-j) k_j^T v_j
// CTA = (32-column block of the state / y, (b,h)); the state block [dk][32]
// stays in shared memory for the whole sequence.  With y null only the state is
// carried (q is not read).
// REV: the anti-causal sum y_n = sum_{m>=n} gamma^(m-n) (q_n . k_m) v_m +
// gamma^(L-n) q_n S_in (S_in: the state after the sequence), walked from the
// last block to the first: for a block at t0 of length l,
//   y_{t0+i} = sum_{j>=i} gamma^(j-i) (q_i.k_j) v_j + gamma^(l-i) q_i S
//   S       <- gamma^l S + sum_{j<l} gamma^j k_j^T v_j
// and state_out is the state at the sequence start.  The backward pass takes
// its two sums that run backwards in time this way.
constexpr int kCF_Cols = 32;
constexpr int kCF_MaxC = 128;

template <bool REV>
__global__ void __launch_bounds__(256)
chunkwise_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                     const float* __restrict__ v, float* __restrict__ y,
                     const float* __restrict__ state_in, float* __restrict__ state_out, int H,
                     int L, int dk, int dv, int C, const __grid_constant__ HeadLog2 hl) {
  extern __shared__ float sm[];
  float* Ss = sm;                          // [dk][32]
  float* Ps = Ss + dk * kCF_Cols;          // [C][C+1]
  float* pw = Ps + C * (C + 1);            // [C+1]: gamma^0 .. gamma^C

  const int bh = blockIdx.y, c0 = blockIdx.x * kCF_Cols, tid = threadIdx.x;
  const float l2g = hl.l2g[bh % H];
  const float* qh = q + (size_t)bh * L * dk;
  const float* kh = k + (size_t)bh * L * dk;
  const float* vh = v + (size_t)bh * L * dv;
  const size_t sbase = (size_t)bh * dk * dv;

  for (int n = tid; n <= C; n += 256) pw[n] = decay_pow(l2g, n);
  for (int e = tid; e < dk * kCF_Cols; e += 256) {
    const int d = e / kCF_Cols, c = e % kCF_Cols;
    Ss[e] = (state_in && c0 + c < dv) ? state_in[sbase + (size_t)d * dv + c0 + c] : 0.f;
  }
  __syncthreads();

  const int n_blk = (L + C - 1) / C;
  for (int bi = 0; bi < n_blk; ++bi) {
    const int t0 = (REV ? n_blk - 1 - bi : bi) * C;
    const int l = min(C, L - t0);
    // 1. decayed, masked scores P[i][j] = gamma^(i-j) q_i.k_j (j <= i; REV:
    // gamma^(j-i), j >= i), for y
    for (int e = tid; y && e < l * l; e += 256) {
      const int i = e / l, j = e % l;
      float s = 0.f;
      if (REV ? j >= i : j <= i) {
        const float* qi = qh + (size_t)(t0 + i) * dk;
        const float* kj = kh + (size_t)(t0 + j) * dk;
        for (int d = 0; d < dk; ++d) s = fmaf(qi[d], kj[d], s);
        s *= pw[REV ? j - i : i - j];
      }
      Ps[i * (C + 1) + j] = s;
    }
    __syncthreads();
    // 2. outputs: intra-block term + decayed cross-block term from the carried
    // state (skipped when only the state is wanted: y null, uniform per CTA)
    for (int e = tid; y && e < l * kCF_Cols; e += 256) {
      const int i = e / kCF_Cols, c = e % kCF_Cols;
      if (c0 + c >= dv) continue;
      float a = 0.f;
      const int j_lo = REV ? i : 0, j_hi = REV ? l - 1 : i;
      for (int j = j_lo; j <= j_hi; ++j) a = fmaf(Ps[i * (C + 1) + j], vh[(size_t)(t0 + j) * dv + c0 + c], a);
      const float* qi = qh + (size_t)(t0 + i) * dk;
      float x = 0.f;
      for (int d = 0; d < dk; ++d) x = fmaf(qi[d], Ss[d * kCF_Cols + c], x);
      y[((size_t)bh * L + t0 + i) * dv + c0 + c] = fmaf(pw[REV ? l - i : i + 1], x, a);
    }
    __syncthreads();
    // 3. state update
    for (int e = tid; e < dk * kCF_Cols; e += 256) {
      const int d = e / kCF_Cols, c = e % kCF_Cols;
      if (c0 + c >= dv) continue;
      float a = pw[l] * Ss[e];
      for (int j = 0; j < l; ++j)
        a = fmaf(pw[REV ? j : l - 1 - j] * kh[(size_t)(t0 + j) * dk + d], vh[(size_t)(t0 + j) * dv + c0 + c], a);
      Ss[e] = a;
    }
    __syncthreads();
  }
  if (state_out) {
    for (int e = tid; e < dk * kCF_Cols; e += 256) {
      const int d = e / kCF_Cols, c = e % kCF_Cols;
      if (c0 + c < dv) state_out[sbase + (size_t)d * dv + c0 + c] = Ss[e];
    }
  }
}

}  // namespace ret
