// chunkwise_wide.cuh -- bf16 chunkwise retention for blocks longer than 128
// (128 < C <= 256, C % 16 == 0) with dk <= 128, on the sm_100a tensor cores.
//
// Same form as chunkwise_tc.cuh (page "Retentive Networks -- Microsoft ...",
// section "Il meccanismo: Multi-Scale Retention": parallel inside a block of
// length C, the state carried from block to block), with the state updated
// once per C tokens.  An M = 128 MMA covers 128 rows, so the block's rows are
// taken as two halves, a = [0, 128) and b = [128, C); the scores of half b
// span every key of the block (the full 128 x 128 piece against the keys of
// half a and the causal piece against its own keys).  One stage; per block the
// MMA warp issues, in order,
//   MMA1a  R  = Q_a K_a^T           N = 128     -> P/O group: Pa~ in place
//   MMA4a  O  = Q_a Sb              N = 128
//   MMA3a  O += Pa~ V_a             K = 128     -> P/O group: y of half a
//   MMA1b  R  = Q_b K^T             N = C       -> P/O group: Pb~ in place
//   MMA4b  O  = Q_b Sb                          (once y of half a is read out)
//   MMA5   S^T += (zeta V)^T K      K = C       -> S group: next Sb
//   MMA3b  O += Pb~ V               K = C       -> P/O group: y of half b
// TMEM: S^T [0, DK), the score region R [DK, DK + 256), O [DK + 256, DK + 384).
// MMAs issued by one thread run in order, so MMA1b overwrites R only after
// MMA3a read Pa~ from it.
//
// Rescaled form (gamma^(C-1) >= 2^-64): V is scaled in place by
// zeta_j / rho (zeta_j = gamma^(l-1-j)), P~ is P masked to j <= i, and
// y_i = gamma^(i+1-l) rho O_i, with the state kept scaled (rho, U) as in the
// dk = 256 kernel.  Direct form (smaller gamma): P~_ij = P_ij gamma^(i-j), O is
// multiplied by xi_i = gamma^(i+1) between MMA4 and MMA3, and the rows of K are
// scaled by zeta once MMA1b has read them, for MMA5.
//
// Decay table: pw[n] = gamma^n, n = 0 .. 256.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "chunkwise_tc.cuh"
#include "tc_common.cuh"

namespace ret {

constexpr uint32_t kCWW_QBox = 256u * 128u;  // Q box: 256 rows of 64 bf16 (rows >= C kept zero)
constexpr uint32_t kCWW_Misc = 1536;         // barriers + pw[0..256]

struct CwWideSmem {
  uint32_t q, k, v, sb, misc, total, kbox;
};

__host__ __device__ inline CwWideSmem cw_wide_smem_plan(int DK, int C) {
  CwWideSmem s;
  s.kbox = (uint32_t)C * 128u;  // K and V boxes: C rows of 64 bf16
  s.q = 0;
  s.k = s.q + (uint32_t)(DK / 64) * kCWW_QBox;
  s.v = s.k + (uint32_t)(DK / 64) * s.kbox;
  s.sb = s.v + 2u * s.kbox;
  s.misc = s.sb + (uint32_t)(DK / 64) * 16384u;
  s.total = s.misc + kCWW_Misc + kSmemAlign;
  return s;
}

template <int DK>
__global__ void __launch_bounds__(kCW_MainThreads, 1)
chunkwise_wide_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                      const __grid_constant__ CUtensorMap mapV, const CwArgs a,
                      const __grid_constant__ CwDecay dec) {
  static_assert(DK == 64 || DK == 128, "dk must be 64 or 128");
  constexpr uint32_t kTmemCols = 512, TM_S = 0, TM_R = DK, TM_O = DK + 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem(smem_raw);
  const int C = a.C;
  const CwWideSmem sp = cw_wide_smem_plan(DK, C);
  uint8_t* sQ = base + sp.q;
  uint8_t* sK = base + sp.k;
  uint8_t* sV = base + sp.v;
  uint8_t* sSb = base + sp.sb;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + sp.misc);
  uint64_t* fullQ = bars + 0;
  uint64_t* fullK = bars + 1;
  uint64_t* fullV = bars + 2;
  uint64_t* emptyQ = bars + 3;    // MMA4b done
  uint64_t* emptyK = bars + 4;    // MMA5 done
  uint64_t* emptyV = bars + 5;    // MMA3b done
  uint64_t* zready = bars + 6;    // V group: V scaled (rescaled) / K scaled (direct)
  // pfull, xdone, pready, mma3done, ofree complete two phases per block (half
  // a, then half b), so parity 0 is half a and parity 1 half b.  Each waiter
  // waits for a before b, and neither half can run a phase ahead of it.
  uint64_t* pfull = bars + 7;     // phases a, b: MMA1a / MMA1b done
  uint64_t* xdone = bars + 8;     // phases a, b: MMA4a / MMA4b done (direct form: xi on O)
  uint64_t* pready = bars + 9;    // phases a, b: P/O group wrote Pa~ / Pb~
  uint64_t* mma3done = bars + 10; // phases a, b: MMA3a / MMA3b done
  uint64_t* ofree = bars + 11;    // phases a, b: O read out
  uint64_t* mma5done = bars + 12; // MMA5 done -> S group
  uint64_t* sready = bars + 13;   // S group: Sb (and the state) ready for the block
  uint64_t* fin = bars + 14;
  uint64_t* p1b = bars + 15;      // MMA1b done -> V group (direct form: K may be scaled)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 16) + 1;
  float* pw = reinterpret_cast<float*>(bars + 17);  // gamma^0 .. gamma^256

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vt = blockIdx.x, bh = blockIdx.y, seg = blockIdx.z;
  const float l2g = dec.l2g[bh % a.H];
  const bool rescaled = (float)(C - 1) * l2g >= -64.f;
  const int n_total = (a.L + C - 1) / C;
  const int c_begin = seg * a.seg_chunks;
  const int c_end = min(c_begin + a.seg_chunks, n_total);
  const int nck = max(c_end - c_begin, 0);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
    mbar_init(zready, 128);
    mbar_init(pfull, 1);
    mbar_init(xdone, 1);
    mbar_init(pready, 128);
    mbar_init(mma3done, 1);
    mbar_init(ofree, 128);
    mbar_init(mma5done, 1);
    mbar_init(sready, 128);
    mbar_init(fin, 1);
    mbar_init(p1b, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int n = threadIdx.x; n <= 256; n += kCW_MainThreads) pw[n] = n == 0 ? 1.f : exp2f((float)n * l2g);
  if (C < 256) {  // rows C..255 of every Q box are read by the half-b MMAs: keep them zero
    const uint32_t rows16 = (256u - (uint32_t)C) * 8u;
    for (uint32_t e = threadIdx.x; e < (uint32_t)(DK / 64) * rows16; e += kCW_MainThreads) {
      const uint32_t b = e / rows16, o = e % rows16;
      *reinterpret_cast<uint4*>(sQ + b * kCWW_QBox + (uint32_t)C * 128u + o * 16u) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nck > 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      const uint32_t qk_bytes = (uint32_t)DK * (uint32_t)C * 2u;
      const uint32_t v_bytes = (uint32_t)kCW_DVT * (uint32_t)C * 2u;
      int issued = 0;
      for (int it = 0; it < nck; ++it) {
        const uint32_t par = (it - 1) & 1;
        const int t0 = (c_begin + it) * C;
        if (it >= 1 && !mbar_wait(emptyQ, par, abort_flag, a.lim)) break;
        mbar_arrive_expect_tx(fullQ, qk_bytes);
        for (int b = 0; b < DK / 64; ++b) tma_load_3d(sQ + b * kCWW_QBox, &mapQ, fullQ, b * 64, t0, bh);
        if (it >= 1 && !mbar_wait(emptyK, par, abort_flag, a.lim)) break;
        if (c_begin + it != a.debug_drop_block) {  // fault injection: a load that never lands
          mbar_arrive_expect_tx(fullK, qk_bytes);
          for (int b = 0; b < DK / 64; ++b) tma_load_3d(sK + b * sp.kbox, &mapK, fullK, b * 64, t0, bh);
        }
        if (it >= 1 && !mbar_wait(emptyV, par, abort_flag, a.lim)) break;
        mbar_arrive_expect_tx(fullV, v_bytes);
        for (int b = 0; b < 2; ++b) tma_load_3d(sV + b * sp.kbox, &mapV, fullV, vt * kCW_DVT + b * 64, t0, bh);
        issued = it + 1;
        if (it + 1 < nck) {  // next block's tiles into L2 while this one runs
          const int tp = t0 + C;
          for (int b = 0; b < DK / 64; ++b) {
            tma_prefetch_l2_3d(&mapQ, b * 64, tp, bh);
            tma_prefetch_l2_3d(&mapK, b * 64, tp, bh);
          }
          for (int b = 0; b < 2; ++b) tma_prefetch_l2_3d(&mapV, vt * kCW_DVT + b * 64, tp, bh);
        }
      }
      if (issued > 0) {
        mbar_drain(fullQ, (issued - 1) & 1, a.lim);
        mbar_drain(fullK, (issued - 1) & 1, a.lim);
        mbar_drain(fullV, (issued - 1) & 1, a.lim);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && nck > 0) {
      const uint32_t id1a = idesc_bf16(128, 128, false, false);
      const uint32_t id1b = idesc_bf16(128, C, false, false);
      const uint32_t id4 = idesc_bf16(128, kCW_DVT, false, false);
      const uint32_t id3 = idesc_bf16(128, kCW_DVT, false, true);
      const uint32_t id5 = idesc_bf16(128, DK, true, true);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aSb = smem_u32(sSb);
      // A = Q rows [row0, row0 + 128), B = K rows (N of them) or Sb, K steps over dk
      auto qk = [&](uint32_t d, uint32_t row0, uint32_t b_base, uint32_t b_box, uint32_t id) {
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aQ + (kk / 4) * kCWW_QBox + row0 * 128u + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b_base + (kk / 4) * b_box + (kk % 4) * 32, 16, 1024);
          mma_ss(d, ad, bd, id, kk > 0);
        }
      };
      // O += R~ V over the first `keys` keys (A = packed P~ in R, B = V rows)
      auto pv = [&](int keys) {
        for (int kk = 0; kk < keys / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(aV + kk * 2048, sp.kbox, 1024);
          mma_ts(tm + TM_O, tm + TM_R + kk * 8, bd, id3, 1);
        }
      };
      for (int it = 0; it < nck; ++it) {
        const uint32_t par = it & 1;
        if (!mbar_wait(fullQ, par, abort_flag, a.lim)) break;
        if (!mbar_wait(fullK, par, abort_flag, a.lim)) break;
        tc_fence_after();
        qk(tm + TM_R, 0, aK, sp.kbox, id1a);  // MMA1a
        mma_commit(pfull);
        if (!mbar_wait(sready, par, abort_flag, a.lim)) break;
        if (!mbar_wait(ofree, 0, abort_flag, a.lim)) break;  // y of the previous half b read out
        tc_fence_after();
        qk(tm + TM_O, 0, aSb, 16384, id4);  // MMA4a
        mma_commit(xdone);
        if (!mbar_wait(rescaled ? zready : fullV, par, abort_flag, a.lim)) break;
        if (!mbar_wait(pready, 0, abort_flag, a.lim)) break;
        tc_fence_after();
        pv(128);  // MMA3a
        mma_commit(mma3done);
        qk(tm + TM_R, 128, aK, sp.kbox, id1b);  // MMA1b
        mma_commit(pfull);
        mma_commit(p1b);
        if (!mbar_wait(ofree, 1, abort_flag, a.lim)) break;  // y of half a read out
        tc_fence_after();
        qk(tm + TM_O, 128, aSb, 16384, id4);  // MMA4b
        mma_commit(xdone);
        mma_commit(emptyQ);
        // MMA5: S^T += (zeta V)^T K (rescaled: zeta on V; direct: zeta on K,
        // scaled by the V group once MMA1b had read K)
        if (!rescaled && !mbar_wait(zready, par, abort_flag, a.lim)) break;
        tc_fence_after();
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aV + kk * 2048, sp.kbox, 1024);
          const uint64_t bd = sdesc_sw128(aK + kk * 2048, sp.kbox, 1024);
          mma_ss(tm + TM_S, ad, bd, id5, 1);
        }
        mma_commit(mma5done);
        mma_commit(emptyK);
        if (!mbar_wait(pready, 1, abort_flag, a.lim)) break;
        tc_fence_after();
        pv(C);  // MMA3b
        mma_commit(mma3done);
        mma_commit(emptyV);
      }
      mma_commit(fin);
      mbar_drain(fin, 0, a.lim);
    }
  } else if (warp >= kWarpZBase) {
    // ---------------------------------------------------- V group (4 warps)
    // Thread t scales rows t and t + 128 (those below C) of V (rescaled form,
    // by zeta_j / rho) or of K (direct form, by zeta_j, after MMA1b).
    const uint32_t t = threadIdx.x - kWarpZBase * 32;
    float rho = cw_rho_first(rescaled, pw[max(min(C, a.L - c_begin * C), 0)]);
    for (int it = 0; it < nck; ++it) {
      const uint32_t par = it & 1;
      const int t0 = (c_begin + it) * C;
      const int l = min(C, a.L - t0);
      if (rescaled) {
        if (!mbar_wait(fullV, par, abort_flag, a.lim)) break;
      } else {
        if (!mbar_wait(fullK, par, abort_flag, a.lim)) break;
        if (!mbar_wait(p1b, par, abort_flag, a.lim)) break;  // MMA1b done: K no longer read unscaled
      }
      const float inv_rho = __frcp_rn(rho);
      for (uint32_t j = t; j < (uint32_t)C; j += 128) {
        const float zeta = ((int)j < l) ? pw[l - 1 - (int)j] : 0.f;
        if (rescaled) {
          scale_row_sw128(sV, j, zeta * inv_rho);
          scale_row_sw128(sV + sp.kbox, j, zeta * inv_rho);
        } else {
          for (int b = 0; b < DK / 64; ++b) scale_row_sw128(sK + b * sp.kbox, j, zeta);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(zready);
      if (it + 1 < nck && rescaled) rho = cw_rho_next(rho, pw[min(C, a.L - t0 - C)]);
    }
  } else if (warp >= kWarpSBase) {
    // ---------------------------------------------------- S group (4 warps)
    // TMEM lane v = this thread's dv column of the state; Sb = bf16 copy
    // (rescaled: of U; direct: of S, with the gamma^l decay applied in TMEM).
    const uint32_t v_loc = threadIdx.x - kWarpSBase * 32;
    const uint32_t lane_off = (uint32_t)((warp - kWarpSBase) * 32) << 16;
    const int v = vt * kCW_DVT + (int)v_loc;
    const size_t dkdv = (size_t)DK * a.dv;
    const float g0 = pw[max(min(C, a.L - c_begin * C), 0)];
    float rho = cw_rho_first(rescaled, g0);
    {
      if (a.n_seg > 1) griddep_wait();  // segment states from the launches before this one
      const float* src = (a.n_seg > 1) ? a.seg_state + ((size_t)bh * a.n_seg + seg) * dkdv
                                       : (a.state_in ? a.state_in + (size_t)bh * dkdv : nullptr);
      const float gu = (rho == 1.f) ? g0 : 1.f;
      const float gc = rescaled ? gu : 1.f;
      for (int d0 = 0; d0 < DK; d0 += 32) {
        float x[32];
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const float sv = src ? src[(size_t)(d0 + u) * a.dv + v] : 0.f;
          x[u] = gc * sv;
          w[u] = __float_as_uint(gu * sv);
        }
        store_row32_sw128(sSb, 16384, v_loc, d0, x);
        tmem_st32(tm + lane_off + TM_S + d0, w);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(sready);
    }
    for (int it = 0; it < nck; ++it) {
      // MMA5 done; MMA4b (the last reader of Sb) ran before it
      if (!mbar_wait(mma5done, it & 1, abort_flag, a.lim)) break;
      tc_fence_after();
      const int t0 = (c_begin + it) * C;
      if (it < nck - 1) {
        const float gn = pw[min(C, a.L - t0 - C)];
        const float rho_n = rescaled ? cw_rho_next(rho, gn) : 1.f;
        const bool write_back = !rescaled || rho_n == 1.f;
        const float mult = rescaled ? gn * rho : gn;
        for (int d0 = 0; d0 < DK; d0 += 32) {
          uint32_t sr[32];
          tmem_ld32(tm + lane_off + TM_S + d0, sr);
          tmem_ld_wait();
          float x[32];
          if (write_back) {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const float sv = __uint_as_float(sr[u]);
              const float sg = mult * sv;
              x[u] = rescaled ? sg : sv;
              sr[u] = __float_as_uint(sg);
            }
            tmem_st32(tm + lane_off + TM_S + d0, sr);
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) x[u] = __uint_as_float(sr[u]);
          }
          store_row32_sw128(sSb, 16384, v_loc, d0, x);
        }
        rho = rho_n;
        if (write_back) tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(sready);
      } else if (a.state_out && seg == a.n_seg - 1) {
        float* so = a.state_out + (size_t)bh * dkdv;
        for (int d0 = 0; d0 < DK; d0 += 32) {
          uint32_t sr[32];
          tmem_ld32(tm + lane_off + TM_S + d0, sr);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) so[(size_t)(d0 + u) * a.dv + v] = rho * __uint_as_float(sr[u]);
        }
      }
    }
  } else {
    // -------------------------------------------------- P/O group (4 warps)
    // TMEM lane r: row r of half a, row 128 + r of half b.
    const int r = (int)threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int row_lo = warp * 32;
    float rho = cw_rho_first(rescaled, pw[max(min(C, a.L - c_begin * C), 0)]);
    mbar_arrive(ofree);  // O starts free
    for (int it = 0; it < nck; ++it) {
      const int t0 = (c_begin + it) * C;
      const int l = min(C, a.L - t0);
      bool ok = true;
      for (int h = 0; h < 2 && ok; ++h) {
        const int i = 128 * h + r;       // row of the block
        const int keys = h ? C : 128;    // columns of R holding scores
        const int diag0 = 128 * h;       // first key of this half's own (causal) piece
        if (!mbar_wait(pfull, (uint32_t)h, abort_flag, a.lim)) { ok = false; break; }
        tc_fence_after();
        // P -> P~ in place (two bf16 per column).  Keys before diag0 are all
        // earlier than every row of the half; keys of the half's own piece
        // are masked to j <= i.
        const uint32_t tp = tm + lane_off + TM_R;
        for (int j0 = 0; j0 < keys; j0 += 32) {
          uint32_t pr[32];
          tmem_ld32(tp + j0, pr);
          tmem_ld_wait();
          uint32_t w[16];
          const int jr = j0 - diag0;  // column relative to the half's own piece
          if (jr >= row_lo + 32) {
#pragma unroll
            for (int u = 0; u < 16; ++u) w[u] = 0u;
          } else if (rescaled) {
            if (jr + 31 <= row_lo) {
#pragma unroll
              for (int u = 0; u < 32; u += 2) w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]), __uint_as_float(pr[u + 1]));
            } else {
#pragma unroll
              for (int u = 0; u < 32; u += 2) {
                const int j = jr + u;
                w[u / 2] = pack_bf16x2((j <= r) ? __uint_as_float(pr[u]) : 0.f,
                                       (j + 1 <= r) ? __uint_as_float(pr[u + 1]) : 0.f);
              }
            }
          } else if (jr + 31 <= row_lo) {
            // whole 32-column piece at or below the diagonal:
            // gamma^(i-j) = gamma^(i-j0-31) * gamma^(31-u)
            const float ar = pw[i - j0 - 31];
#pragma unroll
            for (int u = 0; u < 32; u += 2)
              w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * ar * pw[31 - u],
                                     __uint_as_float(pr[u + 1]) * ar * pw[30 - u]);
          } else {
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              const int j = j0 + u;
              const float f0 = (j <= i) ? pw[i - j] : 0.f;
              const float f1 = (j + 1 <= i) ? pw[i - j - 1] : 0.f;
              w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * f0, __uint_as_float(pr[u + 1]) * f1);
            }
          }
          // For C % 32 == 16 the last piece of half b also reads 16 columns past
          // C (inside R); its packed results land at columns >= C/2, which
          // MMA3b never reads.
          tmem_st16(tp + j0 / 2, w);
        }
        if (!rescaled) {
          // O *= xi_i = gamma^(i+1) once MMA4 wrote Q_h S_prev into O
          if (!mbar_wait(xdone, (uint32_t)h, abort_flag, a.lim)) { ok = false; break; }
          tc_fence_after();
          const float xi = pw[i + 1];
          for (int c0 = 0; c0 < kCW_DVT; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tm + lane_off + TM_O + c0, o);
            tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * xi);
            tmem_st32(tm + lane_off + TM_O + c0, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(pready);
        // y of the half once MMA3 is done: rescaled, y_i = gamma^(i+1-l) rho O_i
        if (!mbar_wait(mma3done, (uint32_t)h, abort_flag, a.lim)) { ok = false; break; }
        tc_fence_after();
        const float yf = rescaled ? exp2f((float)(i + 1 - l) * l2g) * rho : 1.f;
        __nv_bfloat16* wrow0 = a.y + ((size_t)bh * a.L + t0 + 128 * h + row_lo) * a.dv + vt * kCW_DVT;
        uint32_t yb[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tm + lane_off + TM_O + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; ++u)
            yb[c][u] = pack_bf16x2(yf * __uint_as_float(o[2 * u]), yf * __uint_as_float(o[2 * u + 1]));
        }
        tc_fence_before();
        mbar_arrive(ofree);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          store_rows_packed_quad(wrow0 + 32 * c, (size_t)a.dv, lane, yb[c], l - 128 * h - row_lo);
      }
      if (!ok) break;
      if (it + 1 < nck && rescaled) rho = cw_rho_next(rho, pw[min(C, a.L - t0 - C)]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tm, kTmemCols);
  }
}

}  // namespace ret
