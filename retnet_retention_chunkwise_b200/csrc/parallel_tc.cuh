// parallel_tc.cuh -- bf16 parallel-form retention on the sm_100a tensor cores.
//
// y = (Q K^T (.) D) V with D_nm = gamma^(n-m) for m <= n, 0 above the diagonal
// (page "Retentive Networks -- Microsoft ...", section "Il meccanismo", parallel
// form; Eq. (5) / Fig. 2a of the paperhub.cn author responses).  The score
// matrix never reaches HBM.  One CTA owns (b, h, a DVT-column dv slice, DVT = 128,
// or 64 for dv not a multiple of 128) and a
// PAIR of 128-row query tiles, the heaviest with the lightest (qa = n-1-y and
// qb = y), so every CTA walks about the same number of causal key tiles and
// the grid fits in one wave.  For every (query tile, key tile kt <= qt):
//   MMA1  P[pb] = Q K_kt^T     (TMEM, double-buffered)
//   epi   P~ = bf16(P * D) in place, 8 warps (two per TMEM sub-partition, each
//         taking 64 of the 128 key columns)
//   MMA3  O += P~ V_kt        (A from TMEM)
// MMA1 of the next key tile is issued before MMA3 of this one, so the tensor
// core works while the epilogue applies the decay; the MMA warp never waits
// for its own MMAs to finish (they run in issue order), only for the epilogue.  At the end of a query
// tile the epilogue reads O out to y; the second query tile's first MMA3
// waits for that.
//
// Decay without per-element exponentials: for an off-diagonal tile the exponent
// n = 128 (qt - kt) + i - j splits as  i + (128 (qt - kt) - 127) + (127 - j), all
// three parts >= 0, so  gamma^n = pw[i] * T * pw[127 - j]  with one exp2 per tile
// (T) and a 128-entry table; the diagonal tile uses pw[i - j] and the mask.
//
// REV computes the anti-causal sum y_n = sum_{m>=n} gamma^(m-n) (q_n . k_m) v_m
// (the form the backward pass needs for dk and dv, without reversing the
// sequence in memory): key tiles kt >= qt, walked from the last down to the
// diagonal, exponent 128 (kt - qt) + j - i = (127 - i) + (128 (kt - qt) - 127) + j,
// so gamma^n = pw[127 - i] * T * pw[j], and the diagonal tile keeps j >= i.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "chunkwise_tc.cuh"
#include "tc_common.cuh"

namespace ret {

constexpr int kPA_EpiWarps = 8;
constexpr int kPA_WarpProducer = 8;
constexpr int kPA_WarpMma = 9;
constexpr int kPA_Threads = 10 * 32;

struct PaArgs {
  int B, H, L, dv;
  int n_qt;       // query tiles per (b, h)
  int nstages;
  __nv_bfloat16* y;
  WaitLimit lim;
};

struct PaSmem {
  uint32_t q, k, v, misc, total, q_buf, k_stage, v_stage;
};

// Two Q buffers (one per query tile of the pair), NS stages of K and V tiles.
__host__ __device__ inline PaSmem pa_smem_plan(int DK, int DVT, int ns) {
  PaSmem s;
  s.q_buf = (uint32_t)(DK / 64) * 16384u;
  s.k_stage = (uint32_t)(DK / 64) * 16384u;
  s.v_stage = (uint32_t)(DVT / 64) * 16384u;
  s.q = 0;
  s.k = s.q + 2u * s.q_buf;
  s.v = s.k + (uint32_t)ns * s.k_stage;
  s.misc = s.v + (uint32_t)ns * s.v_stage;
  s.total = s.misc + kMiscBytes + kSmemAlign;
  return s;
}

template <int DK, int DVT, bool REV>
__global__ void __launch_bounds__(kPA_Threads, 1)
parallel_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, const PaArgs a,
                   const __grid_constant__ CwDecay dec) {
  static_assert(DK == 64 || DK == 128 || DK == 256, "dk must be 64, 128 or 256");
  static_assert(DVT == 64 || DVT == 128, "dv slice of 64 or 128 columns");
  // TMEM: two P buffers [0, 256), one O accumulator per query tile of the pair
  // [256, 512), so the second tile's MMAs never wait for the first tile's read-out.
  constexpr uint32_t TM_P = 0, TM_O = 256, kTmemCols = 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem(smem_raw);
  const int NS = a.nstages;
  const PaSmem sp = pa_smem_plan(DK, DVT, NS);
  uint8_t* sQ = base + sp.q;
  uint8_t* sK = base + sp.k;
  uint8_t* sV = base + sp.v;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + sp.misc);
  uint64_t* full = bars;          // [4] K, V tile of a stage landed
  uint64_t* empty = bars + 4;     // [4] MMA3 done with the stage
  uint64_t* pfull = bars + 8;     // [2] MMA1 done
  uint64_t* e1done = bars + 12;   // [2] epilogue wrote P~
  uint64_t* qfull = bars + 14;    // [2] Q tile of query tile 0 / 1 landed
  uint64_t* ofull = bars + 16;    // phase t: O of query tile t complete
  uint64_t* fin = bars + 17;      // every MMA issued has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 18) + 1;
  float* pw = reinterpret_cast<float*>(bars + 20);  // gamma^0 .. gamma^128 (16-byte aligned)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vt = blockIdx.x, bh = blockIdx.z;
  // the pair (n-1-y, y): the heavy tile first (forward: the later tile, REV:
  // the earlier one, which has the most key tiles)
  const int qt0 = REV ? (int)blockIdx.y : a.n_qt - 1 - (int)blockIdx.y;
  const int qt1 = REV ? a.n_qt - 1 - (int)blockIdx.y : (int)blockIdx.y;
  const int ntile = (qt0 != qt1) ? 2 : 1;
  auto nkeys = [&](int qt) { return REV ? a.n_qt - qt : qt + 1; };  // key tiles of query tile qt
  const int nk0 = nkeys(qt0);
  const int nitems = nk0 + (ntile == 2 ? nkeys(qt1) : 0);
  const float l2g = dec.l2g[bh % a.H];
  const int cta_id = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  (void)cta_id;
  RET_TRACE_INIT();

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&pfull[i], 1);
      mbar_init(&e1done[i], 32 * kPA_EpiWarps);
      mbar_init(&qfull[i], 1);
    }
    mbar_init(ofull, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int n = threadIdx.x; n <= 128; n += kPA_Threads) pw[n] = n == 0 ? 1.f : exp2f((float)n * l2g);
  if (warp == kPA_WarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  // item i -> (query tile index t in {0,1}, its tile qt, key tile kt); the key
  // tiles of a query tile end with the diagonal one (REV walks them downwards)
  auto item = [&](int i, int& t, int& qt, int& kt) {
    const int k = (i < nk0) ? i : i - nk0;
    t = (i < nk0) ? 0 : 1;
    qt = t ? qt1 : qt0;
    kt = REV ? a.n_qt - 1 - k : k;
  };
  auto first_key = [&](int kt) { return REV ? kt == a.n_qt - 1 : kt == 0; };

  if (warp == kPA_WarpProducer) {
    if (lane == 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      for (int t = 0; t < ntile; ++t) {
        mbar_arrive_expect_tx(&qfull[t], (uint32_t)DK * 128u * 2u);
        for (int b = 0; b < DK / 64; ++b)
          tma_load_3d(sQ + t * sp.q_buf + b * 16384, &mapQ, &qfull[t], b * 64, (t ? qt1 : qt0) * 128, bh);
      }
      const uint32_t bytes = (uint32_t)(DK + DVT) * 128u * 2u;
      int issued = 0;
      for (int i = 0; i < nitems; ++i) {
        int t, qt, kt;
        item(i, t, qt, kt);
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, i, 0);
        mbar_arrive_expect_tx(&full[s], bytes);
        for (int b = 0; b < DK / 64; ++b)
          tma_load_3d(sK + s * sp.k_stage + b * 16384, &mapK, &full[s], b * 64, kt * 128, bh);
        for (int b = 0; b < DVT / 64; ++b)
          tma_load_3d(sV + s * sp.v_stage + b * 16384, &mapV, &full[s], vt * DVT + b * 64, kt * 128, bh);
        issued = i + 1;
      }
      for (int t = 0; t < ntile; ++t) mbar_drain(&qfull[t], 0, a.lim);
      for (int i = max(0, issued - NS); i < issued; ++i) mbar_drain(&full[i % NS], (i / NS) & 1, a.lim);
    }
  } else if (warp == kPA_WarpMma) {
    if (lane == 0) {
      const uint32_t id1 = idesc_bf16(128, 128, false, false);
      const uint32_t id3 = idesc_bf16(128, DVT, false, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = true;
      // O[t] += P~[i] V[i]; the first key tile of a query tile starts O[t]
      // afresh.  The epilogue packs key columns 64c .. 64c+63 of P~ (bf16 pairs)
      // into TMEM columns 64c .. 64c+31, so K step kk reads column
      // 64 (kk / 4) + 8 (kk % 4) of the buffer.
      auto issue_pv = [&](int i) -> bool {
        int t, qt, kt;
        item(i, t, qt, kt);
        const int s = i % NS, pb = i & 1;
        if (!mbar_wait(&e1done[pb], (i >> 1) & 1, abort_flag, a.lim)) return false;
        RET_TRACE_STAMP(cta_id, i, 2);
        tc_fence_after();
        const uint32_t v_s = aV + s * sp.v_stage;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = sdesc_sw128(v_s + kk * 2048, 16384, 1024);
          mma_ts(tm + TM_O + t * 128, tm + TM_P + pb * 128 + (kk / 4) * 64 + (kk % 4) * 8, bd, id3,
                 (!first_key(kt) || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        if (kt == qt) mma_commit(ofull);  // last key tile of this query tile
        return true;
      };
      for (int i = 0; ok && i < nitems; ++i) {
        int t, qt, kt;
        item(i, t, qt, kt);
        const int s = i % NS, pb = i & 1;
        if (first_key(kt) && !mbar_wait(&qfull[t], 0, abort_flag, a.lim)) { ok = false; break; }
        if (!mbar_wait(&full[s], (i / NS) & 1, abort_flag, a.lim)) { ok = false; break; }
        RET_TRACE_STAMP(cta_id, i, 1);
        // P buffer pb was last read by MMA3(i-2), issued before this MMA1 by
        // this thread (MMAs of one thread run in order), and written by the
        // epilogue for item i-2 before that MMA3 was issued: no wait needed.
        tc_fence_after();
        const uint32_t q_s = aQ + t * sp.q_buf, k_s = aK + s * sp.k_stage;
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(q_s + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_s + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          mma_ss(tm + TM_P + pb * 128, ad, bd, id1, kk > 0);
        }
        mma_commit(&pfull[pb]);
        // With two or more stages MMA3 of the previous item follows MMA1 of
        // this one; with one stage the next load waits for this item's MMA3,
        // so MMA3 must come first.
        if (NS >= 2) {
          if (i >= 1 && !issue_pv(i - 1)) { ok = false; break; }
        } else if (!issue_pv(i)) {
          ok = false;
          break;
        }
      }
      if (ok && NS >= 2) issue_pv(nitems - 1);
      mma_commit(fin);
      mbar_drain(fin, 0, a.lim);
    }
  } else {
    // ------------------------------------------------ epilogue (8 warps)
    // Warp w: TMEM lanes 32 (w % 4) .. +31 (rows), key columns 64 (w / 4) .. +63,
    // packed in place into TMEM columns 64 (w / 4) .. +31 of the P buffer (each
    // 32-column read lies at or after the 16 columns written from it, so a
    // warp never overwrites what it has not read yet, and the two warps of a
    // sub-partition touch disjoint columns).
    const int r = (warp & 3) * 32 + lane;  // row of the query tile
    const int row_lo = (warp & 3) * 32;
    const int cbase = (warp >> 2) * 64;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float rowf = pw[REV ? 127 - r : r];
    bool ok = true;
    for (int i = 0; i < nitems; ++i) {
      int t, qt, kt;
      item(i, t, qt, kt);
      const int pb = i & 1;
      if (!mbar_wait(&pfull[pb], (i >> 1) & 1, abort_flag, a.lim)) { ok = false; break; }
      if (threadIdx.x == 0) RET_TRACE_STAMP(cta_id, i, 3);
      tc_fence_after();
      const uint32_t tp = tm + lane_off + TM_P + pb * 128;
      const bool diag = (kt == qt);
      const float rs = diag ? 0.f : rowf * exp2f((float)(128 * (REV ? kt - qt : qt - kt) - 127) * l2g);
      for (int j0 = cbase; j0 < cbase + 64; j0 += 32) {
        uint32_t w[16];
        // diagonal tile: the 32 columns lie wholly on the masked side of row r's warp
        const bool masked = diag && (REV ? j0 + 32 <= row_lo : j0 >= row_lo + 32);
        if (masked) {
#pragma unroll
          for (int u = 0; u < 16; ++u) w[u] = 0u;
        } else {
          uint32_t pr[32];
          tmem_ld32(tp + j0, pr);
          tmem_ld_wait();
          if (!diag && !REV) {
            const float4* cf = reinterpret_cast<const float4*>(pw + 96 - j0);  // pw[127-j] for j = j0+31 .. j0
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const float4 f = cf[7 - q4];  // pw[127-j0-4q4-3 .. 127-j0-4q4]
              w[2 * q4] = pack_bf16x2(__uint_as_float(pr[4 * q4]) * rs * f.w, __uint_as_float(pr[4 * q4 + 1]) * rs * f.z);
              w[2 * q4 + 1] =
                  pack_bf16x2(__uint_as_float(pr[4 * q4 + 2]) * rs * f.y, __uint_as_float(pr[4 * q4 + 3]) * rs * f.x);
            }
          } else if (!diag) {
            const float4* cf = reinterpret_cast<const float4*>(pw + j0);  // pw[j] for j = j0 .. j0+31
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const float4 f = cf[q4];
              w[2 * q4] = pack_bf16x2(__uint_as_float(pr[4 * q4]) * rs * f.x, __uint_as_float(pr[4 * q4 + 1]) * rs * f.y);
              w[2 * q4 + 1] =
                  pack_bf16x2(__uint_as_float(pr[4 * q4 + 2]) * rs * f.z, __uint_as_float(pr[4 * q4 + 3]) * rs * f.w);
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              const int j = j0 + u;
              const float f0 = REV ? ((j >= r) ? pw[j - r] : 0.f) : ((j <= r) ? pw[r - j] : 0.f);
              const float f1 = REV ? ((j + 1 >= r) ? pw[j + 1 - r] : 0.f) : ((j + 1 <= r) ? pw[r - j - 1] : 0.f);
              w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * f0, __uint_as_float(pr[u + 1]) * f1);
            }
          }
        }
        tmem_st16(tp + cbase + (j0 - cbase) / 2, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&e1done[pb]);
      if (threadIdx.x == 0) RET_TRACE_STAMP(cta_id, i, 4);
      if (kt == qt) {
        // query tile complete: O[t] -> y (this warp: its 32 rows, DVT/2 of the columns)
        if (!mbar_wait(ofull, t, abort_flag, a.lim)) { ok = false; break; }
        tc_fence_after();
        const int row0 = qt * 128 + row_lo;
        const int obase = (warp >> 2) * (DVT / 2);
        __nv_bfloat16* wrow0 = a.y + ((size_t)bh * a.L + row0) * a.dv + vt * DVT + obase;
        for (int c0 = 0; c0 < DVT / 2; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tm + lane_off + TM_O + t * 128 + obase + c0, o);
          tmem_ld_wait();
          store_rows_bf16_quad(wrow0 + c0, (size_t)a.dv, lane, o, 1.f, a.L - row0);
        }
        if (threadIdx.x == 0) RET_TRACE_STAMP(cta_id, i, 5);
      }
    }
    (void)ok;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kPA_WarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tm, kTmemCols);
  }
}

}  // namespace ret
