// parallel_tc.cuh -- bf16 parallel-form retention on the sm_100a tensor cores.
//
// y = (Q K^T (.) D) V with D_nm = gamma^(n-m) for m <= n, 0 above the diagonal
// (page "Retentive Networks -- Microsoft ...", section "Il meccanismo", parallel
// form; Eq. (5) / Fig. 2a of the paperhub.cn author responses).  The score
// matrix never reaches HBM: one CTA owns (b, h, a 128-row query tile, a
// 128-column dv slice) and walks the key tiles kt = 0 .. qt (only causal tiles),
//   MMA1  P[pb] = Q K_kt^T    (TMEM, double-buffered)
//   epi   P~ = bf16(P * D) in place
//   MMA3  O += P~ V_kt        (A from TMEM)
// with MMA1 of tile kt+1 issued before MMA3 of tile kt so the tensor core works
// while the epilogue applies the decay.
//
// Decay without per-element exponentials: for an off-diagonal tile the exponent
// n = 128 (qt - kt) + i - j splits as  i + (128 (qt - kt) - 127) + (127 - j), all
// three parts >= 0, so  gamma^n = pw[i] * T * pw[127 - j]  with one exp2 per tile
// (T) and a 128-entry table; the diagonal tile uses pw[i - j] and the mask.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "chunkwise_tc.cuh"
#include "tc_common.cuh"

namespace ret {

struct PaArgs {
  int B, H, L, dv;
  int n_qt;       // query tiles per (b, h)
  int nstages;
  __nv_bfloat16* y;
  WaitLimit lim;
};

struct PaSmem {
  uint32_t q, k, v, misc, total, k_stage, v_stage;
};

__host__ __device__ inline PaSmem pa_smem_plan(int DK, int ns) {
  PaSmem s;
  s.k_stage = (uint32_t)(DK / 64) * 16384u;
  s.v_stage = 2u * 16384u;
  s.q = 0;
  s.k = s.q + (uint32_t)(DK / 64) * 16384u;
  s.v = s.k + (uint32_t)ns * s.k_stage;
  s.misc = s.v + (uint32_t)ns * s.v_stage;
  s.total = s.misc + kMiscBytes + kSmemAlign;
  return s;
}

template <int DK>
__global__ void __launch_bounds__(kCW_Threads, 1)
parallel_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, const PaArgs a,
                   const __grid_constant__ CwDecay dec) {
  static_assert(DK == 64 || DK == 128 || DK == 256, "dk must be 64, 128 or 256");
  constexpr uint32_t TM_P = 0, TM_O = 256, kTmemCols = 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem(smem_raw);
  const int NS = a.nstages;
  const PaSmem sp = pa_smem_plan(DK, NS);
  uint8_t* sQ = base + sp.q;
  uint8_t* sK = base + sp.k;
  uint8_t* sV = base + sp.v;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + sp.misc);
  uint64_t* full = bars;          // [4]
  uint64_t* empty = bars + 4;     // [4]
  uint64_t* pfull = bars + 8;     // [2]
  uint64_t* pfree = bars + 10;    // [2]
  uint64_t* e1done = bars + 12;   // [2]
  uint64_t* qfull = bars + 14;
  uint64_t* ofull = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 16) + 1;
  float* pw = reinterpret_cast<float*>(bars + 17);  // gamma^0 .. gamma^128

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vt = blockIdx.x, qt = a.n_qt - 1 - (int)blockIdx.y, bh = blockIdx.z;
  const float l2g = dec.l2g[bh % a.H];
  const int nkt = qt + 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&pfull[i], 1);
      mbar_init(&pfree[i], 1);
      mbar_init(&e1done[i], 128);
    }
    mbar_init(qfull, 1);
    mbar_init(ofull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int n = threadIdx.x; n <= 128; n += kCW_Threads) pw[n] = n == 0 ? 1.f : exp2f((float)n * l2g);
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      mbar_arrive_expect_tx(qfull, (uint32_t)DK * 128u * 2u);
      for (int b = 0; b < DK / 64; ++b) tma_load_3d(sQ + b * 16384, &mapQ, qfull, b * 64, qt * 128, bh);
      const uint32_t bytes = (uint32_t)(DK + 128) * 128u * 2u;
      int issued = 0;
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % NS;
        if (kt >= NS && !mbar_wait(&empty[s], ((kt / NS) - 1) & 1, abort_flag, a.lim)) break;
        mbar_arrive_expect_tx(&full[s], bytes);
        for (int b = 0; b < DK / 64; ++b)
          tma_load_3d(sK + s * sp.k_stage + b * 16384, &mapK, &full[s], b * 64, kt * 128, bh);
        for (int b = 0; b < 2; ++b)
          tma_load_3d(sV + s * sp.v_stage + b * 16384, &mapV, &full[s], vt * 128 + b * 64, kt * 128, bh);
        issued = kt + 1;
      }
      mbar_drain(qfull, 0, a.lim);
      for (int kt = max(0, issued - NS); kt < issued; ++kt) mbar_drain(&full[kt % NS], (kt / NS) & 1, a.lim);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t id1 = idesc_bf16(128, 128, false, false);
      const uint32_t id3 = idesc_bf16(128, 128, false, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = mbar_wait(qfull, 0, abort_flag, a.lim);
      // O += P~[kt] V[kt]
      auto issue_pv = [&](int kt) -> bool {
        const int s = kt % NS, pb = kt & 1;
        if (!mbar_wait(&e1done[pb], (kt >> 1) & 1, abort_flag, a.lim)) return false;
        tc_fence_after();
        const uint32_t v_s = aV + s * sp.v_stage;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = sdesc_sw128(v_s + kk * 2048, 16384, 1024);
          mma_ts(tm + TM_O, tm + TM_P + pb * 128 + kk * 8, bd, id3, (kt > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&pfree[pb]);
        mma_commit(&empty[s]);
        return true;
      };
      for (int kt = 0; ok && kt < nkt; ++kt) {
        const int s = kt % NS, pb = kt & 1;
        if (!mbar_wait(&full[s], (kt / NS) & 1, abort_flag, a.lim)) { ok = false; break; }
        if (kt >= 2 && !mbar_wait(&pfree[pb], ((kt >> 1) - 1) & 1, abort_flag, a.lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_s = aK + s * sp.k_stage;
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aQ + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_s + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          mma_ss(tm + TM_P + pb * 128, ad, bd, id1, kk > 0);
        }
        mma_commit(&pfull[pb]);
        // With two or more stages, MMA3 of the previous tile follows MMA1 of this
        // one.  With a single stage the next tile's load waits for this tile's
        // MMA3, so MMA3 must come first.
        if (NS >= 2) {
          if (kt >= 1 && !issue_pv(kt - 1)) { ok = false; break; }
        } else if (!issue_pv(kt)) {
          ok = false;
          break;
        }
      }
      if (ok && NS >= 2) issue_pv(nkt - 1);
      mma_commit(ofull);
      mbar_drain(ofull, 0, a.lim);
    }
  } else {
    const uint32_t r = threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float rowf = pw[r];
    bool ok = true;
    for (int kt = 0; kt < nkt; ++kt) {
      const int pb = kt & 1;
      if (!mbar_wait(&pfull[pb], (kt >> 1) & 1, abort_flag, a.lim)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tp = tm + lane_off + TM_P + pb * 128;
      const bool diag = (kt == qt);
      const float rs = diag ? 0.f : rowf * exp2f((float)(128 * (qt - kt) - 127) * l2g);
      for (int j0 = 0; j0 < 128; j0 += 32) {
        uint32_t pr[32];
        tmem_ld32(tp + j0, pr);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < 32; u += 2) {
          const int j = j0 + u;
          float f0, f1;
          if (diag) {
            f0 = (j <= (int)r) ? pw[r - j] : 0.f;
            f1 = (j + 1 <= (int)r) ? pw[r - j - 1] : 0.f;
          } else {
            f0 = rs * pw[127 - j];
            f1 = rs * pw[126 - j];
          }
          w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * f0, __uint_as_float(pr[u + 1]) * f1);
        }
        tmem_st16(tp + j0 / 2, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&e1done[pb]);
    }
    if (ok && mbar_wait(ofull, 0, abort_flag, a.lim)) {
      tc_fence_after();
      const int row = qt * 128 + (int)r;
      __nv_bfloat16* yrow = a.y + ((size_t)bh * a.L + row) * a.dv + vt * 128;
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tm + lane_off + TM_O + c0, o);
        tmem_ld_wait();
        if (row < a.L) {
          uint4* dst = reinterpret_cast<uint4*>(yrow + c0);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * q4 + 0]), __uint_as_float(o[8 * q4 + 1]));
            w.y = pack_bf16x2(__uint_as_float(o[8 * q4 + 2]), __uint_as_float(o[8 * q4 + 3]));
            w.z = pack_bf16x2(__uint_as_float(o[8 * q4 + 4]), __uint_as_float(o[8 * q4 + 5]));
            w.w = pack_bf16x2(__uint_as_float(o[8 * q4 + 6]), __uint_as_float(o[8 * q4 + 7]));
            dst[q4] = w;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tm, kTmemCols);
  }
}

}  // namespace ret
