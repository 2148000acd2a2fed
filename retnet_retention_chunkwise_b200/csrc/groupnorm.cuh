// groupnorm.cuh -- per-head group normalisation of the retention output.
//
// One normalisation group per head (author responses on paperhub.cn,
// "Retentive Network: A Successor to Transformer for Large Language Models",
// reply comparing GroupNorm with LayerNorm: heads carry different statistics).
// For each (b, h, n) the dv values of y_n are one group:
//     out_c = (y_c - mean) / sqrt(var + eps) * w[h*dv + c] + bias[h*dv + c]
// with the biased variance, and w, bias optional (null: 1 and 0).
//
// An optional output gate follows (same page, reply on the "transformer without
// softmax" remark: gated multi-scale retention, no formula given).  Reading:
//     out_c *= act(g_c),  act = identity, swish x sigmoid(x), or sigmoid(x)
// with g a gate input of y's shape.
//
// This kernel runs on a finished y (one warp per row, fp32 statistics in two
// passes over registers): it reads y (and g) once and writes the output once,
// so it is bound by HBM.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace ret {

constexpr int kGN_MaxDv = 1024;
constexpr int kGN_RowsPerBlock = 8;

template <typename T>
__device__ __forceinline__ void gn_load4(const T* p, float (&x)[4]);
template <>
__device__ __forceinline__ void gn_load4<float>(const float* p, float (&x)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  x[0] = v.x, x[1] = v.y, x[2] = v.z, x[3] = v.w;
}
template <>
__device__ __forceinline__ void gn_load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  x[0] = __uint_as_float(v.x << 16), x[1] = __uint_as_float(v.x & 0xffff0000u);
  x[2] = __uint_as_float(v.y << 16), x[3] = __uint_as_float(v.y & 0xffff0000u);
}
template <typename T>
__device__ __forceinline__ void gn_store4(T* p, const float (&x)[4]);
template <>
__device__ __forceinline__ void gn_store4<float>(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
template <>
__device__ __forceinline__ void gn_store4<__nv_bfloat16>(__nv_bfloat16* p, const float (&x)[4]) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
  uint2 v;
  v.x = *reinterpret_cast<const uint32_t*>(&a);
  v.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = v;
}

// 8 bf16 (16 bytes) at once
__device__ __forceinline__ void gn_load8(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void gn_store8(__nv_bfloat16* p, const float (&x)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

enum GateAct { kGateNone = 0, kGateSwish = 1, kGateSigmoid = 2 };

// sigmoid through the fast exponential and divide (a few ulp; the result is
// rounded to the output dtype next).  -x is capped at 80 so that 1 + e^-x stays
// finite and far below the divide's 2^126 range limit; sigmoid(-80) = 1.8e-35.
__device__ __forceinline__ float gate_act(float x, int act) {
  if (act == kGateNone) return x;
  const float sg = __fdividef(1.f, 1.f + __expf(fminf(-x, 80.f)));
  return act == kGateSwish ? x * sg : sg;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Value e (0..7) of 8 bf16 packed in a uint4.
__device__ __forceinline__ float bf8_at(const uint4& v, int e) {
  const uint32_t w = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
  return __uint_as_float((e & 1) ? (w & 0xffff0000u) : (w << 16));
}

// bf16 rows with dv % 256 == 0: each lane keeps its 8 values per step (and
// the gate's) as the packed 16-byte words it loaded, and widens them where
// they are used; half the registers of fp32 copies, so more rows are resident
// per SM and more loads are in flight.
template <int STEPS, bool GATE>
__device__ __forceinline__ void groupnorm_row_bf16x8(const __nv_bfloat16* yr, __nv_bfloat16* orow, int lane,
                                                     int dv, float eps, const float* wr, const float* br,
                                                     const __nv_bfloat16* gr, int act) {
  uint4 xv[STEPS], gv[GATE ? STEPS : 1];
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int c = (i * 32 + lane) * 8;
    xv[i] = make_uint4(0, 0, 0, 0);
    if (c < dv) {
      xv[i] = *reinterpret_cast<const uint4*>(yr + c);
      if constexpr (GATE) gv[i] = *reinterpret_cast<const uint4*>(gr + c);
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < STEPS; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) s += bf8_at(xv[i], e);  // zeros past dv
  const float mean = warp_sum(s) / (float)dv;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    if ((i * 32 + lane) * 8 < dv) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = bf8_at(xv[i], e) - mean;
        q += d * d;
      }
    }
  }
  const float rstd = rsqrtf(warp_sum(q) / (float)dv + eps);
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int c = (i * 32 + lane) * 8;
    if (c < dv) {
      float z[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        z[e] = (bf8_at(xv[i], e) - mean) * rstd;
        if (wr) z[e] *= wr[c + e];
        if (br) z[e] += br[c + e];
      }
      if constexpr (GATE) {
#pragma unroll
        for (int e = 0; e < 8; ++e) z[e] *= gate_act(bf8_at(gv[i], e), act);
      }
      gn_store8(orow + c, z);
    }
  }
}

// One warp per (b, h, n) row.  Vectorised (VEC values per lane per step: 8
// for bf16 when dv % 256 == 0, 4 when dv % 128 == 0), else one value per lane
// per step; STEPS steps cover dv (<= 1024), so the row lives in VEC * STEPS
// registers per lane (x2 with the gate; packed bf16 words for VEC = 8).  out
// may alias y.  GATE: act(gate) multiplies the result.
// Packed bf16 rows of up to 512 values fit in 40 registers a thread, six
// blocks of 8 rows per SM (the gated form needs that bound to get there).
template <typename T, int VEC, int STEPS, bool GATE>
__global__ void __launch_bounds__(32 * kGN_RowsPerBlock, (VEC == 8 && STEPS <= 2) ? 6 : 1)
groupnorm_rows_kernel(const T* y, T* out, long long rows, int H, int L, int dv, float eps,
                      const float* __restrict__ w, const float* __restrict__ bias, const T* __restrict__ gate,
                      int act) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kGN_RowsPerBlock + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int h = (int)((row / L) % H);
  const T* yr = y + row * dv;
  const T* gr = GATE ? gate + row * dv : nullptr;
  T* orow = out + row * dv;
  if constexpr (VEC == 8) {
    groupnorm_row_bf16x8<STEPS, GATE>(yr, orow, lane, dv, eps, w ? w + (size_t)h * dv : nullptr,
                                      bias ? bias + (size_t)h * dv : nullptr, gr, act);
    return;
  }
  float x[STEPS][VEC], gv[GATE ? STEPS : 1][VEC];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int c = (i * 32 + lane) * VEC;
#pragma unroll
    for (int e = 0; e < VEC; ++e) x[i][e] = 0.f;
    if (c < dv) {
      // the gate values are loaded here, with y, so both reads are in flight together
      if constexpr (VEC == 8) {
        gn_load8(yr + c, x[i]);
        if constexpr (GATE) gn_load8(gr + c, gv[i]);
      } else if constexpr (VEC == 4) {
        gn_load4<T>(yr + c, x[i]);
        if constexpr (GATE) gn_load4<T>(gr + c, gv[i]);
      } else {
        x[i][0] = (float)yr[c];
        if constexpr (GATE) gv[i][0] = (float)gr[c];
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) s += x[i][e];
    }
  }
  const float mean = warp_sum(s) / (float)dv;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    if ((i * 32 + lane) * VEC < dv) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float d = x[i][e] - mean;
        q += d * d;
      }
    }
  }
  const float rstd = rsqrtf(warp_sum(q) / (float)dv + eps);
  const float* wr = w ? w + (size_t)h * dv : nullptr;
  const float* br = bias ? bias + (size_t)h * dv : nullptr;
#pragma unroll
  for (int i = 0; i < STEPS; ++i) {
    const int c = (i * 32 + lane) * VEC;
    if (c < dv) {
      float z[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        z[e] = (x[i][e] - mean) * rstd;
        if (wr) z[e] *= wr[c + e];
        if (br) z[e] += br[c + e];
      }
      if constexpr (GATE) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) z[e] *= gate_act(gv[i][e], act);
      }
      if constexpr (VEC == 8) {
        gn_store8(orow + c, z);
      } else if constexpr (VEC == 4) {
        gn_store4<T>(orow + c, z);
      } else {
        orow[c] = (T)z[0];
      }
    }
  }
}

// Launch with the fewest steps (a power of two) that cover dv.
template <typename T, int VEC, bool GATE, int STEPS = 1>
void launch_groupnorm_rows(unsigned blocks, cudaStream_t st, const T* y, T* out, long long rows, int H, int L,
                           int dv, float eps, const float* w, const float* b, const T* gate, int act) {
  constexpr int kMax = kGN_MaxDv / (32 * VEC);
  if constexpr (STEPS < kMax) {
    if (dv > 32 * VEC * STEPS) {
      launch_groupnorm_rows<T, VEC, GATE, 2 * STEPS>(blocks, st, y, out, rows, H, L, dv, eps, w, b, gate, act);
      return;
    }
  }
  groupnorm_rows_kernel<T, VEC, STEPS, GATE>
      <<<blocks, 32 * kGN_RowsPerBlock, 0, st>>>(y, out, rows, H, L, dv, eps, w, b, gate, act);
}

}  // namespace ret
