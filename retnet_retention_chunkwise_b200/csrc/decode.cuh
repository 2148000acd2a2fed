// decode.cuh -- one recurrent (decode) step, in place on the fp32 state:
//     S <- gamma_h S + k^T v ;  y = q S
// (page "Retentive Networks -- Microsoft ...", section "Il meccanismo:
// Multi-Scale Retention", recurrent form).
//
// The step streams the whole state once in and once out (2 * dk * dv * 4 bytes
// per head) and does 4 flops per state element, so it is bound by HBM.  Design:
//  * one CTA = one (b, h) and a block of 128 state columns; 8 warps;
//  * lane l owns columns [4l, 4l+4) of the block: a warp covers one 512-byte
//    row segment with one 128-bit load and one 128-bit store per row
//    (coalesced), rows d = warp, warp+8, ... are walked with 4 rows in flight;
//  * q and k are staged in shared memory as fp32 (broadcast reads);
//  * the readout y = q S sums each warp's rows in registers and the 8 warp
//    partials through shared memory.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace ret {

constexpr int kDecodeThreads = 256;
constexpr int kDecodeCols = 128;     // state columns per CTA
constexpr int kDecodeMaxDk = 1024;

struct HeadGamma {
  float g[1024];  // per-head decay (RET_MAX_HEADS)
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f32(float* p, float x) { *p = x; }
__device__ __forceinline__ void from_f32(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T, bool kVec>
__global__ void __launch_bounds__(kDecodeThreads)
recurrent_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      T* __restrict__ y, float* __restrict__ S, int H, int dk, int dv,
                      const __grid_constant__ HeadGamma hg) {
  __shared__ float sq[kDecodeMaxDk];
  __shared__ float sk[kDecodeMaxDk];
  __shared__ float4 red[kDecodeThreads / 32][32];

  const int bh = blockIdx.y;
  const float g = hg.g[bh % H];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * kDecodeCols + lane * 4;

  for (int i = threadIdx.x; i < dk; i += kDecodeThreads) {
    sq[i] = to_f32(q[(size_t)bh * dk + i]);
    sk[i] = to_f32(k[(size_t)bh * dk + i]);
  }
  float vv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
    vv[u] = (col + u < dv) ? to_f32(v[(size_t)bh * dv + col + u]) : 0.f;
  __syncthreads();

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float* Sh = S + (size_t)bh * dk * dv;
  if (kVec) {
    // dv % 4 == 0 and S 16-byte aligned: whole float4 columns, col < dv or not at all.
    if (col < dv) {
      int d = warp;
      for (; d + 24 < dk; d += 32) {
        float4 s[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          s[u] = *reinterpret_cast<const float4*>(Sh + (size_t)(d + 8 * u) * dv + col);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float kd = sk[d + 8 * u], qd = sq[d + 8 * u];
          s[u].x = fmaf(g, s[u].x, kd * vv[0]);
          s[u].y = fmaf(g, s[u].y, kd * vv[1]);
          s[u].z = fmaf(g, s[u].z, kd * vv[2]);
          s[u].w = fmaf(g, s[u].w, kd * vv[3]);
          *reinterpret_cast<float4*>(Sh + (size_t)(d + 8 * u) * dv + col) = s[u];
          acc[0] = fmaf(qd, s[u].x, acc[0]);
          acc[1] = fmaf(qd, s[u].y, acc[1]);
          acc[2] = fmaf(qd, s[u].z, acc[2]);
          acc[3] = fmaf(qd, s[u].w, acc[3]);
        }
      }
      for (; d < dk; d += 8) {
        float4 s = *reinterpret_cast<const float4*>(Sh + (size_t)d * dv + col);
        const float kd = sk[d], qd = sq[d];
        s.x = fmaf(g, s.x, kd * vv[0]);
        s.y = fmaf(g, s.y, kd * vv[1]);
        s.z = fmaf(g, s.z, kd * vv[2]);
        s.w = fmaf(g, s.w, kd * vv[3]);
        *reinterpret_cast<float4*>(Sh + (size_t)d * dv + col) = s;
        acc[0] = fmaf(qd, s.x, acc[0]);
        acc[1] = fmaf(qd, s.y, acc[1]);
        acc[2] = fmaf(qd, s.z, acc[2]);
        acc[3] = fmaf(qd, s.w, acc[3]);
      }
    }
  } else {
    for (int d = warp; d < dk; d += 8) {
      const float kd = sk[d], qd = sq[d];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (col + u < dv) {
          float* p = Sh + (size_t)d * dv + col + u;
          const float s = fmaf(g, *p, kd * vv[u]);
          *p = s;
          acc[u] = fmaf(qd, s, acc[u]);
        }
      }
    }
  }
  red[warp][lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  if (warp == 0) {
    float4 t = red[0][lane];
#pragma unroll
    for (int w = 1; w < kDecodeThreads / 32; ++w) {
      const float4 o = red[w][lane];
      t.x += o.x;
      t.y += o.y;
      t.z += o.z;
      t.w += o.w;
    }
    const float r[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (col + u < dv) from_f32(y + (size_t)bh * dv + col + u, r[u]);
  }
}

// Small grids (few heads, e.g. batch 1): a block of 32 state columns per CTA,
// one column per lane (a warp still reads one 128-byte row segment per load),
// so that the grid has four times as many CTAs to spread the state stream over
// the SMs; eight rows in flight per warp.
constexpr int kDecodeNarrowCols = 32;

template <typename T>
__global__ void __launch_bounds__(kDecodeThreads)
recurrent_step_narrow_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                             T* __restrict__ y, float* __restrict__ S, int H, int dk, int dv,
                             const __grid_constant__ HeadGamma hg) {
  __shared__ float sq[kDecodeMaxDk];
  __shared__ float sk[kDecodeMaxDk];
  __shared__ float red[kDecodeThreads / 32][32];

  const int bh = blockIdx.y;
  const float g = hg.g[bh % H];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = blockIdx.x * kDecodeNarrowCols + lane;

  for (int i = threadIdx.x; i < dk; i += kDecodeThreads) {
    sq[i] = to_f32(q[(size_t)bh * dk + i]);
    sk[i] = to_f32(k[(size_t)bh * dk + i]);
  }
  const float vv = (col < dv) ? to_f32(v[(size_t)bh * dv + col]) : 0.f;
  __syncthreads();

  float acc = 0.f;
  float* Sh = S + (size_t)bh * dk * dv;
  if (col < dv) {
    int d = warp;
    for (; d + 56 < dk; d += 64) {
      float s[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) s[u] = Sh[(size_t)(d + 8 * u) * dv + col];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        s[u] = fmaf(g, s[u], sk[d + 8 * u] * vv);
        Sh[(size_t)(d + 8 * u) * dv + col] = s[u];
        acc = fmaf(sq[d + 8 * u], s[u], acc);
      }
    }
    for (; d < dk; d += 8) {
      const float sv = fmaf(g, Sh[(size_t)d * dv + col], sk[d] * vv);
      Sh[(size_t)d * dv + col] = sv;
      acc = fmaf(sq[d], sv, acc);
    }
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float t = red[0][lane];
#pragma unroll
    for (int w = 1; w < kDecodeThreads / 32; ++w) t += red[w][lane];
    if (col < dv) from_f32(y + (size_t)bh * dv + col, t);
  }
}

}  // namespace ret
