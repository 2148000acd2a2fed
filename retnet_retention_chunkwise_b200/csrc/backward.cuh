// backward.cuh -- pieces of the backward passes around the three retention sums.
//
// With y_n = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m (page "Retentive Networks
// -- Microsoft ...", section "Il meccanismo: Multi-Scale Retention") and an
// upstream gradient dy, the chain rule gives three sums of the same kind:
//     dq_n = sum_{m<=n} gamma^(n-m) (dy_n . v_m) k_m     = retention(dy, v, k)_n
//     dk_m = sum_{n>=m} gamma^(n-m) (v_m . dy_n) q_n     = retention_rev(v, dy, q)_m
//     dv_m = sum_{n>=m} gamma^(n-m) (k_m . q_n) dy_n     = retention_rev(k, q, dy)_m
// The last two run backwards in time (anti-causal); the parallel and chunkwise
// kernels take them directly (their REV instantiations walk the key tiles or
// blocks from the end), so the backward pass is three launches of the forward
// kernels with no copy of the inputs.
//
// A carried state (state_in S0, state_out S_out with upstream gradient dS_out)
// adds, from y_n += gamma^(n+1) q_n S0 and S_out = gamma^L S0 +
// sum_m gamma^(L-1-m) k_m^T v_m:
//     dq_n += gamma^(n+1) dy_n S0^T
//     dk_m += gamma^(L-1-m) v_m dS_out^T,   dv_m += gamma^(L-1-m) k_m dS_out
//     dS0   = gamma^L dS_out + sum_n gamma^(n+1) q_n^T dy_n
// Each is the initial-state term of one of the three sums: the anti-causal sum
// started from S_in adds gamma^(L-m) a_m S_in, and gamma^(L-1-m) =
// gamma^(L-m) / gamma, so
//     dq = retention(dy, v, k;         state_in S0^T)
//     dk = retention_rev(v, dy, q;     state_in (dS_out / gamma)^T)
//     dv = retention_rev(k, q, dy;     state_in dS_out / gamma)
// and the last sum's state_out T = sum_n gamma^n q_n^T dy_n + gamma^(L-1)
// dS_out gives dS0 = gamma T.  Heads whose gamma is below kBwdMinGamma take a
// zero initial state in the dk and dv sums instead (1 / gamma would overflow):
// bwd_last_token_kernel adds the m = L-1 row's term (gamma^0 = 1) and
// bwd_finish_state_kernel the gamma^L dS_out of dS0.  The terms dropped are
// the dS_out terms of dk_m and dv_m for m < L-1, whose factor gamma^(L-1-m) is
// below kBwdMinGamma.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "decode.cuh"  // HeadGamma

namespace ret {

constexpr float kBwdMinGamma = 8.673617379884035e-19f;  // 2^-60

// Initial states of the three sums, one 32 x 32 tile of one (b, h) per block
// (grid: ceil(dv/32), ceil(dk/32), B*H; block 32 x 8).  s0, dso [BH][dk][dv]
// (either may be null: no output from it); s0t, x2 [BH][dv][dk], x3
// [BH][dk][dv].
__global__ void __launch_bounds__(256) bwd_state_prep_kernel(const float* __restrict__ s0,
                                                             const float* __restrict__ dso,
                                                             float* __restrict__ s0t, float* __restrict__ x2,
                                                             float* __restrict__ x3, int H, int dk, int dv,
                                                             const __grid_constant__ HeadGamma hg) {
  __shared__ float ts[32][33], td[32][33];
  const long long bh = blockIdx.z;
  const float g = hg.g[bh % H];
  const bool small = !(g >= kBwdMinGamma);
  const int j0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  const size_t base = (size_t)bh * dk * dv;
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + threadIdx.x;
    if (i < dk && j < dv) {
      const size_t e = base + (size_t)i * dv + j;
      if (s0) ts[r][threadIdx.x] = s0[e];
      if (dso) {
        const float x = small ? 0.f : dso[e] / g;
        td[r][threadIdx.x] = x;
        x3[e] = x;
      }
    }
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int j = j0 + r, i = i0 + threadIdx.x;
    if (i < dk && j < dv) {
      const size_t e = base + (size_t)j * dk + i;
      if (s0) s0t[e] = ts[threadIdx.x][r];
      if (dso) x2[e] = td[threadIdx.x][r];
    }
  }
}

template <typename T>
__device__ __forceinline__ float bwd_ld(const T* p) {
  return static_cast<float>(*p);
}
template <>
__device__ __forceinline__ float bwd_ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// For heads with gamma < kBwdMinGamma: dk_{L-1} += v_{L-1} dS_out^T and
// dv_{L-1} += k_{L-1} dS_out, one (b, h) per block (grid B*H, 256 threads);
// other heads return at once.
template <typename T>
__global__ void __launch_bounds__(256) bwd_last_token_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                             const float* __restrict__ dso, T* dkk, T* dvv,
                                                             int H, int L, int dk, int dv,
                                                             const __grid_constant__ HeadGamma hg) {
  const long long bh = blockIdx.x;
  if (hg.g[bh % H] >= kBwdMinGamma) return;
  const T* kr = k + ((size_t)bh * L + (L - 1)) * dk;
  const T* vr = v + ((size_t)bh * L + (L - 1)) * dv;
  T* dkr = dkk + ((size_t)bh * L + (L - 1)) * dk;
  T* dvr = dvv + ((size_t)bh * L + (L - 1)) * dv;
  const float* D = dso + (size_t)bh * dk * dv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // dk row: one warp per component i, lanes across j
  for (int i = warp; i < dk; i += 8) {
    float acc = 0.f;
    for (int j = lane; j < dv; j += 32) acc += D[(size_t)i * dv + j] * bwd_ld(vr + j);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dkr[i] = static_cast<T>(bwd_ld(dkr + i) + acc);
  }
  // dv row: one thread per component j, walking i (rows of D read coalesced)
  for (int j = threadIdx.x; j < dv; j += 256) {
    float acc = 0.f;
    for (int i = 0; i < dk; ++i) acc += bwd_ld(kr + i) * D[(size_t)i * dv + j];
    dvr[j] = static_cast<T>(bwd_ld(dvr + j) + acc);
  }
}

// dS0 = gamma_h T + gL_h dS_out over [BH][dk][dv], where gL_h = gamma_h^L for
// heads below kBwdMinGamma (their T was taken from a zero initial state) and 0
// otherwise.  out may alias t or dso (each element is read before it is
// written, by the same thread); dso may be null.
__global__ void __launch_bounds__(256) bwd_finish_state_kernel(const float* t, const float* dso, float* out,
                                                               long long BH, int H, int per_head,
                                                               const __grid_constant__ HeadGamma hg,
                                                               const __grid_constant__ HeadGamma gl) {
  const long long total = BH * per_head;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int h = (int)((e / per_head) % H);
    float r = hg.g[h] * t[e];
    if (dso) r += gl.g[h] * dso[e];
    out[e] = r;
  }
}

}  // namespace ret
