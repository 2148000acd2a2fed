// chunkwise_tc.cuh -- bf16 chunkwise retention on the sm_100a tensor cores.
//
// The form (page "Retentive Networks -- Microsoft ...", section "Il meccanismo:
// Multi-Scale Retention": blocks of length C, parallel inside a block,
// recurrence between blocks), written out for a block of length l at t0:
//   P   = Q_c K_c^T                                   (scores, l x l)
//   O   = (P (.) D) V_c  +  diag(xi) Q_c S_prev        D_ij = gamma^(i-j), j <= i
//   S   = gamma^l S_prev + K_c^T diag(zeta) V_c        xi_i = gamma^(i+1), zeta_j = gamma^(l-1-j)
//
// One CTA owns (b, h, a 128-column slice of dv, a run of consecutive blocks)
// and walks its blocks in order with the fp32 state slice resident in TMEM,
// held transposed (lanes = the 128 dv columns, columns = dk) so the state
// update has M = 128 for every dk.  Warp roles (448 threads, both kernels):
//   warps 0-3    P/O group: TMEM lane r = row r of the block.  P -> P~ in place
//                (bf16 pairs), xi on O in the direct form; y out in the dk = 256
//                kernel.
//   warps 4-7    S group: the state copy Sb for the next block's cross term
//                (and the state rescale when it is due), state_out.
//   warps 8-11   V group: zeta on the rows of V (rescaled form) or of K, or
//                (zeta V)^T in TMEM (direct form); y out in the dk <= 128
//                kernel; in the dk = 256 kernel it also keeps half of the state.
//   warp 12      TMA producer: Q, K, V of each block on their own barriers.
//   warp 13      TMEM allocator; lane 0 issues every tcgen05.mma.
//
// Two forms of the decay (chosen per head, uniform over the CTA):
//   rescaled (gamma^(C-1) >= 2^-64): V scaled by zeta_j / rho, P~ = P masked
//     to j <= i, y_i = gamma^(i+1-l) rho O_i.  The state is kept scaled: TMEM
//     holds U with the decayed state rho U, and U is multiplied through only
//     when rho would drop below 2^-64 (cw_rho_next).
//   direct (smaller gamma): P~_ij = P_ij gamma^(i-j), O scaled by xi after the
//     cross term, the state decayed by gamma^l in TMEM each block.
//
// chunkwise_tc_kernel<DK> (DK 64, 128; NS = 2..4 stages, O double-buffered):
//   MMA1  P[pb] = Q K^T            A = Q  (smem, K-major)   B = K  (smem, K-major)
//   MMA5  S^T  += (zeta V)^T K     A = V  (smem, MN-major, or TMEM)  B = K (smem, MN-major)
//   MMA4  O     = Q Sb             A = Q  (smem, K-major)   B = Sb (smem, K-major)
//   MMA3  O    += P~ V             A = P~ (TMEM, bf16)      B = V  (smem, MN-major)
//   TMEM: S^T [0, DK), P [DK, DK + 128), O buffers [DK + 128, DK + 384): block
//   it uses O buffer it % 2, so MMA4 of the next block does not wait for the
//   read-out of this block's y, which the V group does while the P/O group
//   turns the next block's P into P~.
// chunkwise_tc256_kernel (DK = 256, one stage): the scores and the cross term
// in one N = C + 128 MMA, [P | X] = Q [K ; Sb]^T, then the state update and
// P~ V (see there).
//
// Decay factors come from a per-CTA table pw[n] = gamma^n, n = 0..128 (exp2 of
// n*log2(gamma), gamma^0 = 1): the intra-block mask uses pw[i-j], xi = pw[i+1],
// zeta = pw[l-1-j], the state decay pw[l].  Only the y factor of the rescaled
// form has a negative exponent, bounded by the same 2^-64 test.
//
// Long sequences with few (b, h) are split into segments run by separate CTAs:
// chunk_state_kernel computes each segment's decayed K^T V sum, state_scan_kernel
// turns those into every segment's initial state, and the main kernel starts
// each segment from its own state.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include "tc_common.cuh"

namespace ret {

constexpr int kCW_Threads = 192;      // helper kernels: 4 epilogue warps, TMA warp, MMA warp
constexpr int kCW_DVT = 128;          // dv columns per CTA
// Main chunkwise kernel warp roles (448 threads).
constexpr int kWarpSBase = 4;         // warps 4-7: state group
constexpr int kWarpZBase = 8;         // warps 8-11: (zeta V)^T builder
constexpr int kWarpProducer = 12;     // TMA producer
constexpr int kWarpMma = 13;          // TMEM allocator + MMA issuer
constexpr int kCW_MainThreads = 14 * 32;
constexpr int kCW_MaxStages = 4;
constexpr uint32_t kSmemAlign = 1024;
constexpr uint32_t kMiscBytes = 1024;

struct CwDecay {
  float l2g[1024];  // per-head log2(gamma); -inf for gamma = 0 (RET_MAX_HEADS)
};

struct CwArgs {
  int B, H, L, dv, C;
  int seg_chunks;           // blocks per segment
  int n_seg;                // segments per (b, h)
  int nstages;
  __nv_bfloat16* y;
  const float* state_in;    // initial state when n_seg == 1 (may be null = zeros)
  float* state_out;         // may be null
  const float* seg_state;   // [BH][n_seg][dk][dv] initial states when n_seg > 1
  // Anti-causal sums (REV) only, dk <= 128 kernel: when set (and seg_state is
  // null), segment g starts from the transpose of the state in slot
  // seg_tr_step * (g + 1) - 1 (the last segment: slot seg_tr_nseg - 1) of
  // seg_tr, laid out [BH][seg_tr_nseg][dv][dk]: the scanned segment states of
  // an anti-causal sum whose state is the transpose of this one.
  const float* seg_tr;
  int seg_tr_nseg, seg_tr_step;
  // Causal dk <= 128 kernel with one 128-column dv slice per head, built
  // with GN: the per-head group normalisation of each y row in the epilogue,
  // before the store, with eps and the optional per-channel weight and bias
  // [H][dv].
  float gn_eps;
  const float* gn_w;
  const float* gn_b;
  WaitLimit lim;
  int debug_drop_block;     // fault injection: block whose K load is never issued (-1 = none)
};

struct CwSmem {
  uint32_t q, k, v, sb, misc, total;
  uint32_t q_stage, k_stage, v_stage;
};

// Shared-memory plan (byte offsets from a 1024-aligned base).  Q stages keep
// 128 rows per 64-column box so the M = 128 MMA reads only zeros past row C.
__host__ __device__ inline CwSmem cw_smem_plan(int DK, int C, int ns) {
  CwSmem s;
  s.q_stage = (uint32_t)(DK / 64) * 128u * 128u;
  s.k_stage = (uint32_t)(DK / 64) * (uint32_t)C * 128u;
  s.v_stage = 2u * (uint32_t)C * 128u;
  s.q = 0;
  s.k = s.q + (uint32_t)ns * s.q_stage;
  s.v = s.k + (uint32_t)ns * s.k_stage;
  s.sb = s.v + (uint32_t)ns * s.v_stage;
  s.misc = s.sb + (uint32_t)(DK / 64) * 128u * 128u;
  s.total = s.misc + kMiscBytes + kSmemAlign;  // + slack for aligning the base
  return s;
}

__device__ __forceinline__ uint8_t* align_smem(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + (kSmemAlign - 1)) &
                                    ~uintptr_t(kSmemAlign - 1));
}

// Waits that ignore the abort flag (time-bounded only): used at teardown to
// drain copies and MMAs still in flight before the CTA releases its memory.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, WaitLimit lim) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy, lim);
}

// Scale the 128-byte row r of a 128B-swizzled bf16 tile in place by f.
__device__ __forceinline__ void scale_row_sw128(uint8_t* tile, uint32_t r, float f) {
  // all eight loads first, so the row costs one shared-memory round trip
  uint4 w[8];
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) w[c] = *reinterpret_cast<const uint4*>(tile + sw128_off(r, c));
#pragma unroll
  for (uint32_t c = 0; c < 8; ++c) {
    w[c].x = pack_bf16x2(bf16lo_to_f32(w[c].x) * f, bf16hi_to_f32(w[c].x) * f);
    w[c].y = pack_bf16x2(bf16lo_to_f32(w[c].y) * f, bf16hi_to_f32(w[c].y) * f);
    w[c].z = pack_bf16x2(bf16lo_to_f32(w[c].z) * f, bf16hi_to_f32(w[c].z) * f);
    w[c].w = pack_bf16x2(bf16lo_to_f32(w[c].w) * f, bf16hi_to_f32(w[c].w) * f);
    *reinterpret_cast<uint4*>(tile + sw128_off(r, c)) = w[c];
  }
}

// Write 32 floats as bf16 into row r, columns [c0, c0+32) of a 128B-swizzled
// tile made of 64-column boxes of `box_bytes` bytes each.
__device__ __forceinline__ void store_row32_sw128(uint8_t* tile, uint32_t box_bytes, uint32_t r,
                                                  uint32_t c0, const float* x) {
  uint8_t* box = tile + (c0 / 64) * box_bytes;
  const uint32_t ch0 = (c0 % 64) / 8;
#pragma unroll
  for (uint32_t q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(x[8 * q + 0], x[8 * q + 1]);
    w.y = pack_bf16x2(x[8 * q + 2], x[8 * q + 3]);
    w.z = pack_bf16x2(x[8 * q + 4], x[8 * q + 5]);
    w.w = pack_bf16x2(x[8 * q + 6], x[8 * q + 7]);
    *reinterpret_cast<uint4*>(box + sw128_off(r, ch0 + q)) = w;
  }
}

// Store 32 columns of 32 rows (one row per lane, 32 fp32 each, scaled by f)
// as bf16 with fewer memory transactions: a 4x4 transpose of 16-byte pieces
// inside each lane quad (two shuffle stages) makes every store instruction
// write 8 rows x 64 contiguous bytes instead of 32 rows x 16 bytes.
// `row0` points at column c0 of the warp's first row; rows with
// (lane-row >= nrows) are not written.
__device__ __forceinline__ void store_rows_quad_core(__nv_bfloat16* row0, size_t row_stride, int lane,
                                                     uint32_t (&c)[4][4], int nrows) {
  const bool b0 = lane & 1, b1 = lane & 2;
#pragma unroll
  for (int k = 0; k < 4; k += 2)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, b0 ? c[k][e] : c[k + 1][e], 1);
      if (b0) c[k][e] = recv; else c[k + 1][e] = recv;
    }
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, b1 ? c[k][e] : c[k + 2][e], 2);
      if (b1) c[k][e] = recv; else c[k + 2][e] = recv;
    }
  // lane = 4m + p now holds piece p (columns 8p..8p+7) of rows 4m .. 4m+3
  const int m = lane >> 2, p = lane & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int row = 4 * m + k;
    if (row < nrows)
      *reinterpret_cast<uint4*>(row0 + (size_t)row * row_stride + 8 * p) = make_uint4(c[k][0], c[k][1], c[k][2], c[k][3]);
  }
}

__device__ __forceinline__ void store_rows_bf16_quad(__nv_bfloat16* row0, size_t row_stride, int lane,
                                                     const uint32_t (&o)[32], float f, int nrows) {
  uint32_t c[4][4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e)
      c[k][e] = pack_bf16x2(f * __uint_as_float(o[8 * k + 2 * e]), f * __uint_as_float(o[8 * k + 2 * e + 1]));
  store_rows_quad_core(row0, row_stride, lane, c, nrows);
}

// Same, from 32 columns already packed as bf16 pairs (w[u] = columns 2u, 2u+1).
__device__ __forceinline__ void store_rows_packed_quad(__nv_bfloat16* row0, size_t row_stride, int lane,
                                                       const uint32_t (&w)[16], int nrows) {
  uint32_t c[4][4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int e = 0; e < 4; ++e) c[k][e] = w[4 * k + e];
  store_rows_quad_core(row0, row_stride, lane, c, nrows);
}

// Scaled state (rescaled form): TMEM holds U, and the state decayed for the
// coming block is rho * U.  After a block rho takes on gamma^l of the next
// block instead of the state being multiplied in TMEM; only when rho would
// drop below 2^-64 is U multiplied through (and rho reset to 1), so the
// scaled operands (zeta V / rho, U) stay below 2^64 in magnitude.
__device__ __forceinline__ float cw_rho_next(float rho, float gl) {
  const float r = gl * rho;
  return r < 0x1p-64f ? 1.f : r;
}

// rho for the first block of a segment (g0 = gamma^l0): 1 in the direct form.
__device__ __forceinline__ float cw_rho_first(bool rescaled, float g0) {
  return (rescaled && g0 >= 0x1p-64f) ? g0 : 1.f;
}

template <int DK, bool REV, bool GN = false>
__global__ void __launch_bounds__(kCW_MainThreads, 1)
chunkwise_tc_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapY,
                    const CwArgs a, const __grid_constant__ CwDecay dec) {
  static_assert(DK == 64 || DK == 128 || DK == 256, "dk must be 64, 128 or 256");
  // TMEM: S^T [0, DK), P [DK, DK + 128), two O buffers of 128 columns after
  // it, so the next block's MMA4 never waits for this block's y read-out.
  constexpr uint32_t TM_S = 0, TM_P = DK, TM_O = DK + 128;
  constexpr uint32_t kTmemCols = 512;
  static_assert(DK + 3 * 128 <= (int)kTmemCols, "TMEM plan");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem(smem_raw);
  const int C = a.C, NS = a.nstages;
  const CwSmem sp = cw_smem_plan(DK, C, NS);
  uint8_t* sQ = base + sp.q;
  uint8_t* sK = base + sp.k;
  uint8_t* sV = base + sp.v;
  uint8_t* sSb = base + sp.sb;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + sp.misc);
  uint64_t* fullQ = bars;          // [4] TMA -> MMA
  uint64_t* fullK = bars + 4;      // [4] TMA -> MMA
  uint64_t* fullV = bars + 8;      // [4] TMA -> V group, MMA
  uint64_t* emptyQ = bars + 12;    // [4] MMA4 done -> producer
  uint64_t* emptyK = bars + 16;    // [4] MMA5 done -> producer
  uint64_t* zready = bars + 24;    // [4] V group: scaled V (K) of stage s written -> MMA5 (MMA1)
  uint64_t* pfull = bars + 28;     // MMA1 done -> P/O group
  uint64_t* mma3done = bars + 30;  // [2] per O buffer: MMA3 done -> V group (y)
  uint64_t* ocross = bars + 32;    // MMA5 + MMA4 done -> P/O group, S group
  uint64_t* pready = bars + 33;    // P/O group: P~ (and xi O) written -> MMA3
  uint64_t* sready = bars + 35;    // S group: state copy + rescaled state written -> MMA5, MMA4
  uint64_t* ofree = bars + 36;     // [2] per O buffer: V group read y out -> MMA4 two blocks later
  uint64_t* fin = bars + 38;       // teardown drain of the MMA pipe
  uint64_t* ystaged = bars + 41;   // [4] V group: y of the block staged -> producer (TMA store)
  uint64_t* emptyV = bars + 45;    // [4] MMA3 done -> producer (y staged in the Q buffer)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 39);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 39) + 1;
  float* pw = reinterpret_cast<float*>(bars + 52);  // gamma^0 .. gamma^128
  // y of a block is staged for its TMA store in a buffer that is dead after
  // MMA3: the block's Q buffer when it holds a C x 128 bf16 tile (DK = 128),
  // so that the V buffer can be reloaded as soon as MMA3 is done, else the
  // block's V buffer.
  constexpr bool kYinQ = DK >= 128;
  // Rescaled form at dk = 64: zeta / rho goes on the rows of K (half the bytes
  // of V's rows) as soon as K lands, before MMA1, so that P = Q (zeta K)^T
  // carries it into P~ V and V stays as loaded; MMA5 takes V and zeta K.
  // Elsewhere it goes on V's rows.
  constexpr bool kZetaK = DK == 64;
  const uint32_t y_box = kYinQ ? 16384u : (uint32_t)C * 128u;  // bytes between the two 64-column boxes of y

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vt = blockIdx.x, bh = blockIdx.y, seg = blockIdx.z;
  const float l2g = dec.l2g[bh % a.H];
  // Rescaled form (see the file header) when gamma^(C-1) >= 2^-64; else the
  // direct form.  Uniform over the CTA (one head).
  const bool rescaled = (float)(C - 1) * l2g >= -64.f;
  const bool zeta_k = kZetaK && rescaled;
  const int n_total = (a.L + C - 1) / C;
  const int c_begin = seg * a.seg_chunks;
  const int c_end = min(c_begin + a.seg_chunks, n_total);
  const int nck = max(c_end - c_begin, 0);
  // Step it of the walk takes block blk_idx(it): forward from the segment's
  // first block, REV (the anti-causal sum) from its last block down.
  auto blk_idx = [&](int it) { return REV ? c_end - 1 - it : c_begin + it; };
  auto blk_t0 = [&](int it) { return blk_idx(it) * C; };
  auto blk_len = [&](int it) { return min(C, a.L - blk_t0(it)); };
  const int l_first = nck > 0 ? blk_len(0) : 0;
  const int cta_id = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  (void)cta_id;
  RET_TRACE_INIT();
  if (threadIdx.x == 0) RET_TRACE_STAMP(cta_id, 255, 0);  // trace: kernel entry

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&fullQ[i], 1);
      mbar_init(&fullK[i], 1);
      mbar_init(&fullV[i], 1);
      mbar_init(&emptyQ[i], 1);
      mbar_init(&emptyK[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&zready[i], 128);
    mbar_init(pfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&mma3done[i], 1);
      mbar_init(&ofree[i], 128);
    }
    mbar_init(ocross, 1);
    mbar_init(pready, 128);
    mbar_init(sready, 128);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&ystaged[i], 128);
      mbar_init(&emptyV[i], 1);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int n = threadIdx.x; n <= 128; n += kCW_MainThreads) pw[n] = n == 0 ? 1.f : exp2f((float)n * l2g);
  if (C < 128) {  // rows C..127 of every Q box are read by the M = 128 MMA: keep them zero
    const uint32_t rows16 = (128u - (uint32_t)C) * 8u;  // 16-byte pieces per box
    const uint32_t per_stage = (uint32_t)(DK / 64) * rows16;
    for (uint32_t e = threadIdx.x; e < (uint32_t)NS * per_stage; e += kCW_MainThreads) {
      const uint32_t s = e / per_stage, rem = e % per_stage;
      const uint32_t b = rem / rows16, o = rem % rows16;
      *reinterpret_cast<uint4*>(sQ + s * sp.q_stage + b * 16384u + (uint32_t)C * 128u + o * 16u) =
          make_uint4(0, 0, 0, 0);
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
  if (threadIdx.x == 0) RET_TRACE_STAMP(cta_id, 255, 1);  // trace: prologue done

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ producer
    // Q, K, V of each block go to their own stage buffers with their own
    // barriers, so each is reloaded as soon as its last reader is done: K
    // after MMA5, V after MMA3, and the buffer that stages y (Q or V) after
    // the TMA stores of that y have read it.
    // The next block's tiles are prefetched into L2 as soon as this block's
    // loads are issued, so a reload waits on L2 rather than on DRAM.
    if (lane == 0 && nck > 0) {
      tma_prefetch_desc(&mapQ);
      tma_prefetch_desc(&mapK);
      tma_prefetch_desc(&mapV);
      const uint32_t qk_bytes = (uint32_t)DK * (uint32_t)C * 2u;
      const uint32_t v_bytes = (uint32_t)kCW_DVT * (uint32_t)C * 2u;
      for (int it = 0; it < min(NS, nck); ++it) {
        const int t0 = blk_t0(it);
        for (int b = 0; b < DK / 64; ++b) {
          tma_prefetch_l2_3d(&mapK, b * 64, t0, bh);
          tma_prefetch_l2_3d(&mapQ, b * 64, t0, bh);
        }
        for (int b = 0; b < 2; ++b) tma_prefetch_l2_3d(&mapV, vt * kCW_DVT + b * 64, t0, bh);
      }
      int issued = 0;
      for (int it = 0; it < nck; ++it) {
        const int s = it % NS;
        const uint32_t par = ((it / NS) - 1) & 1;
        const int t0 = blk_t0(it);
        if (it >= NS && !mbar_wait(&emptyK[s], par, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, it, 0);
        if (blk_idx(it) != a.debug_drop_block) {  // fault injection: a load that never lands
          mbar_arrive_expect_tx(&fullK[s], qk_bytes);
          for (int b = 0; b < DK / 64; ++b)
            tma_load_3d(sK + s * sp.k_stage + b * C * 128, &mapK, &fullK[s], b * 64, t0, bh);
        }
        // The staging buffer of stage s holds y of block it - NS (staged after
        // MMA3): store it with two TMA tensor stores, and reload the buffer
        // once they have read it.
        uint8_t* ys = kYinQ ? sQ + s * sp.q_stage : sV + s * sp.v_stage;
        auto store_y = [&]() -> bool {
          if (!mbar_wait(&ystaged[s], par, abort_flag, a.lim)) return false;
          const int ty = blk_t0(it - NS);
          tma_store_3d(&mapY, ys, vt * kCW_DVT, ty, bh);
          tma_store_3d(&mapY, ys + y_box, vt * kCW_DVT + 64, ty, bh);
          bulk_commit_group();
          bulk_wait_read_all();
          return true;
        };
        auto load_q = [&]() {
          mbar_arrive_expect_tx(&fullQ[s], qk_bytes);
          for (int b = 0; b < DK / 64; ++b)
            tma_load_3d(sQ + s * sp.q_stage + b * 16384, &mapQ, &fullQ[s], b * 64, t0, bh);
        };
        auto load_v = [&]() {
          mbar_arrive_expect_tx(&fullV[s], v_bytes);
          for (int b = 0; b < 2; ++b)
            tma_load_3d(sV + s * sp.v_stage + b * C * 128, &mapV, &fullV[s], vt * kCW_DVT + b * 64, t0, bh);
        };
        if (kYinQ) {
          // V after MMA3 of block it - NS; Q after y of that block left its buffer
          if (it >= NS && !mbar_wait(&emptyV[s], par, abort_flag, a.lim)) break;
          load_v();
          if (it >= NS && !store_y()) break;
          load_q();
        } else {
          if (it >= NS && !mbar_wait(&emptyQ[s], par, abort_flag, a.lim)) break;
          load_q();
          if (it >= NS && !store_y()) break;
          load_v();
        }
        issued = it + 1;
        if (it + NS < nck) {
          const int tp = blk_t0(it + NS);
          for (int b = 0; b < DK / 64; ++b) {
            tma_prefetch_l2_3d(&mapK, b * 64, tp, bh);
            tma_prefetch_l2_3d(&mapQ, b * 64, tp, bh);
          }
          for (int b = 0; b < 2; ++b) tma_prefetch_l2_3d(&mapV, vt * kCW_DVT + b * 64, tp, bh);
        }
      }
      // y of the last blocks (those no later load had to wait for)
      if (issued == nck) {
        for (int j = max(0, nck - NS); j < nck; ++j) {
          if (!mbar_wait(&ystaged[j % NS], (j / NS) & 1, abort_flag, a.lim)) break;
          const uint8_t* ys = kYinQ ? sQ + (j % NS) * sp.q_stage : sV + (j % NS) * sp.v_stage;
          tma_store_3d(&mapY, ys, vt * kCW_DVT, blk_t0(j), bh);
          tma_store_3d(&mapY, ys + y_box, vt * kCW_DVT + 64, blk_t0(j), bh);
          bulk_commit_group();
        }
      }
      bulk_wait_all();  // the y stores issued by this thread are complete
      RET_TRACE_STAMP(cta_id, 255, 3);  // trace: last y store complete
      // every load issued must land before the CTA may exit
      for (int it = max(0, issued - NS); it < issued; ++it) {
        mbar_drain(&fullQ[it % NS], (it / NS) & 1, a.lim);
        mbar_drain(&fullK[it % NS], (it / NS) & 1, a.lim);
        mbar_drain(&fullV[it % NS], (it / NS) & 1, a.lim);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------- MMA issuer
    // Order per block: MMA1 (P = Q K^T), MMA5 (state update; frees K), MMA4
    // (Q S into O buffer it % 2; frees Q), MMA3 (P~ V).  MMAs issued by one
    // thread run in order, so MMA1 of the next block overwrites P only after
    // MMA3 has read P~, and MMA4 overwrites an O buffer only after MMA5 has
    // read (zeta V)^T from it.
    if (lane == 0 && nck > 0) {
      const uint32_t id1 = idesc_bf16(128, C, false, false);
      const uint32_t id4 = idesc_bf16(128, kCW_DVT, false, false);
      const uint32_t id3 = idesc_bf16(128, kCW_DVT, false, true);
      const uint32_t id5 = idesc_bf16(128, DK, rescaled, true);  // A = V^T (smem, MN-major) or TMEM
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aSb = smem_u32(sSb);
      for (int it = 0; it < nck; ++it) {
        const int s = it % NS, ob = it & 1;
        const uint32_t par = (it / NS) & 1;
        const uint32_t t_o = tm + TM_O + 128u * (uint32_t)ob;
        if (!mbar_wait4(&fullK[s], par, &fullQ[s], par, zeta_k ? &zready[s] : &fullQ[s], par, &fullQ[s], par,
                        abort_flag, a.lim))
          break;
        RET_TRACE_STAMP(cta_id, it, 1);
        tc_fence_after();
        const uint32_t q_s = aQ + s * sp.q_stage, k_s = aK + s * sp.k_stage, v_s = aV + s * sp.v_stage;
        // MMA1: P = Q K^T
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(q_s + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_s + (kk / 4) * C * 128 + (kk % 4) * 32, 16, 1024);
          mma_ss(tm + TM_P, ad, bd, id1, kk > 0);
        }
        mma_commit(pfull);
        RET_TRACE_STAMP(cta_id, it, 14);
        // MMA5: S^T += (zeta V)^T K, onto the state already rescaled by gamma^l.
        // Rescaled form: zeta sits on the V tile (or on the K tile at dk = 64)
        // in place, V read MN-major from shared memory.  Direct form:
        // (zeta V)^T was built in the columns of this block's (free) O buffer.
        // zready is per stage: in the rescaled form the V group runs ahead by up
        // to NS blocks, so one barrier could complete two phases unobserved.
        // (with zeta on K nothing else has waited for this block's V tile: MMA5
        // and MMA3 read it, so wait for its load here).  The wait for MMA4's O
        // buffer (y of block it - 2 read out of it) goes with these.
        if (!mbar_wait4(zeta_k ? &fullV[s] : &zready[s], par, sready, it & 1, &ofree[ob], (it >> 1) & 1, sready,
                        it & 1, abort_flag, a.lim))
          break;
        RET_TRACE_STAMP(cta_id, it, 2);
        tc_fence_after();
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(k_s + kk * 2048, C * 128, 1024);
          if (rescaled)
            mma_ss(tm + TM_S, sdesc_sw128(v_s + kk * 2048, C * 128, 1024), bd, id5, 1);
          else
            mma_ts(tm + TM_S, t_o + kk * 8, bd, id5, 1);
        }
        mma_commit(&emptyK[s]);
        // MMA4: O = Q S_copy into buffer ob (y of block it - 2 has left it)
        RET_TRACE_STAMP(cta_id, it, 11);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(q_s + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(aSb + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          mma_ss(t_o, ad, bd, id4, kk > 0);
        }
        mma_commit(ocross);
        mma_commit(&emptyQ[s]);
        // MMA3: O += P~ V
        if (!mbar_wait(pready, it & 1, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, it, 4);
        tc_fence_after();
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(v_s + kk * 2048, C * 128, 1024);
          mma_ts(t_o, tm + TM_P + kk * 8, bd, id3, 1);
        }
        mma_commit(&mma3done[ob]);
        if (kYinQ) mma_commit(&emptyV[s]);
        RET_TRACE_STAMP(cta_id, it, 15);
      }
      mma_commit(fin);
      mbar_drain(fin, 0, a.lim);
    }
  } else if (warp >= kWarpZBase) {
    // ---------------------------------------------------- V group (4 warps)
    // Two jobs, one block apart: zeta for block it + 1 (on V in the rescaled
    // form, (zeta V)^T into that block's O buffer in the direct form), then y
    // of block it out of its O buffer once MMA3 is done.  TMEM lane t = dv
    // column t for (zeta V)^T, row t of the block for y.
    const uint32_t t = threadIdx.x - kWarpZBase * 32;
    const uint32_t lane_off = (uint32_t)((warp - kWarpZBase) * 32) << 16;
    const int row_lo = (warp - kWarpZBase) * 32;
    float rho_z = cw_rho_first(rescaled, pw[l_first]);  // rho of the block zeta is applied to
    float rho_y = rho_z;                                 // rho of the block read out
    mbar_arrive(&ofree[0]);  // both O buffers start free
    mbar_arrive(&ofree[1]);
    auto zeta_step = [&](int it) -> bool {
      const int s = it % NS;
      if (!mbar_wait(zeta_k ? &fullK[s] : &fullV[s], (it / NS) & 1, abort_flag, a.lim)) return false;
      if (t == 0) RET_TRACE_STAMP(cta_id, it, 13);
      const int l = min(C, a.L - blk_t0(it));
      uint8_t* vs = sV + s * sp.v_stage;
      if (zeta_k) {
        // row j of the K tile (one 64-column box) scaled in place by zeta_j / rho
        const float rinv = __frcp_rn(rho_z);
        if (RET_BC(s < NS, 105)) {
          for (int j = (int)t; j < C; j += 128) {
            const float zs = ((j < l) ? pw[REV ? j : l - 1 - j] : 0.f) * rinv;
            scale_row_sw128(sK + s * sp.k_stage, (uint32_t)j, zs);
          }
        }
        fence_proxy_async_smem();
      } else if (rescaled) {
        // row j of the V tile scaled in place by zeta_j = gamma^(l-1-j) (0 past
        // the end), divided by rho.  C = 128: thread t takes both 64-column
        // boxes of row t, one after the other (sixteen loads in flight were
        // slower); shorter blocks spread (row, box) over all threads.
        const float rinv = __frcp_rn(rho_z);
        if (RET_BC(s < NS, 105)) {
          if (C == 128) {
            const float zs = (((int)t < l) ? pw[REV ? (int)t : l - 1 - (int)t] : 0.f) * rinv;
            scale_row_sw128(vs, t, zs);
            scale_row_sw128(vs + C * 128, t, zs);
          } else {
            for (int w = (int)t; w < 2 * C; w += 128) {
              const int j = w % C;
              const float zs = ((j < l) ? pw[REV ? j : l - 1 - j] : 0.f) * rinv;
              scale_row_sw128(vs + (w / C) * C * 128, (uint32_t)j, zs);
            }
          }
        }
        fence_proxy_async_smem();
      } else {
        // (zeta V)^T into the block's O buffer (its y of two blocks before was
        // read out by this group already): lane v holds column v of V scaled
        // row-wise by zeta_j, two rows per 32-bit column.  V is read from its
        // swizzled tile as 32-bit pairs (v0, v0+1) of rows j and j+1 and
        // re-paired by a byte permute.
        const uint32_t vb = t / 64, vv = t % 64;
        const uint32_t vchunk = vv / 8;                // 16-byte chunk of the row
        const uint32_t vbyte = ((vv % 8) & ~1u) * 2u;  // byte of the pair (v0, v0+1): 0, 4, 8, 12
        const uint32_t sel = (t & 1) ? 0x7632u : 0x5410u;
        const uint8_t* vt_s = vs + vb * C * 128;
        const uint32_t t_o = tm + lane_off + TM_O + 128u * (uint32_t)(it & 1);
        for (int j0 = 0; j0 < C; j0 += 32) {
          uint32_t w[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const uint32_t j = (uint32_t)j0 + 2u * u;
            if (!RET_BC(j + 1 < (uint32_t)C + 16u, 106)) break;
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(vt_s + j * 128 + ((vchunk ^ (j & 7)) << 4) + vbyte);
            const uint32_t w1 =
                *reinterpret_cast<const uint32_t*>(vt_s + (j + 1) * 128 + ((vchunk ^ ((j + 1) & 7)) << 4) + vbyte);
            const uint32_t pr = __byte_perm(w0, w1, sel);
            const float z0 = ((int)j < l) ? pw[REV ? (int)j : l - 1 - (int)j] : 0.f;
            const float z1 = ((int)j + 1 < l) ? pw[REV ? (int)j + 1 : l - 2 - (int)j] : 0.f;
            w[u] = pack_bf16x2(bf16lo_to_f32(pr) * z0, bf16hi_to_f32(pr) * z1);
          }
          // When C % 32 == 16 the last piece covers 16 rows past C (zeta = 0
          // there, read from the next, allocated, part of shared memory); the
          // results land in columns MMA5 never reads.
          tmem_st16(t_o + j0 / 2, w);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      mbar_arrive(&zready[s]);
      if (t == 0) RET_TRACE_STAMP(cta_id, it, 3);
      if (it + 1 < nck && rescaled) rho_z = cw_rho_next(rho_z, pw[blk_len(it + 1)]);
      return true;
    };
    // y = (gamma^(r+1-l) rho in the rescaled form) O, staged in the block's Q
    // or V buffer (dead after MMA3, not reloaded before the producer stored y
    // out of it) for two TMA tensor stores by the producer.
    auto y_step = [&](int it) -> bool {
      const int s = it % NS, ob = it & 1;
      if (!mbar_wait(&mma3done[ob], (it >> 1) & 1, abort_flag, a.lim)) return false;
      if (t == 0) RET_TRACE_STAMP(cta_id, it, 9);
      tc_fence_after();
      const int l = blk_len(it);
      const int r = (int)t;
      const float yf = rescaled ? exp2f((float)(REV ? -r : r + 1 - l) * l2g) * rho_y : 1.f;
      if (it + 1 < nck && rescaled) rho_y = cw_rho_next(rho_y, pw[blk_len(it + 1)]);
      uint8_t* ystage = kYinQ ? sQ + s * sp.q_stage : sV + s * sp.v_stage;
      const uint32_t t_o = tm + lane_off + TM_O + 128u * (uint32_t)ob;
      // Group normalisation of the row (the head's whole dv), with y = yf * o
      // for the accumulator row o: the mean and biased variance of o from
      // one pass over the row in TMEM (sums shifted by the row's first value,
      // eight partial sums to keep the dependent chains short), scaled by yf;
      // then z = o * (yf rstd) - mean rstd in the second pass.
      float gn_a = 1.f, gn_b = 0.f;
      if constexpr (GN) {
        float sh = 0.f, s1[8], s2[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) s1[j] = 0.f, s2[j] = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < kCW_DVT; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(t_o + c0, o);
          tmem_ld_wait();
          if (c0 == 0) sh = __uint_as_float(o[0]);
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const float d = __uint_as_float(o[u]) - sh;
            s1[u & 7] += d;
            s2[u & 7] = fmaf(d, d, s2[u & 7]);
          }
        }
#pragma unroll
        for (int j = 1; j < 8; ++j) s1[0] += s1[j], s2[0] += s2[j];
        const float m1 = s1[0] * (1.f / kCW_DVT);
        const float var = fmaxf(s2[0] * (1.f / kCW_DVT) - m1 * m1, 0.f) * (yf * yf);
        const float rstd = rsqrtf(var + a.gn_eps);
        gn_a = yf * rstd;
        gn_b = -(sh + m1) * gn_a;
      }
#pragma unroll
      for (int c0 = 0; c0 < kCW_DVT; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(t_o + c0, o);
        tmem_ld_wait();
        float x[32];
        if constexpr (GN) {
#pragma unroll
          for (int u = 0; u < 32; ++u) x[u] = fmaf(__uint_as_float(o[u]), gn_a, gn_b);
          const int ch = (bh % a.H) * kCW_DVT + c0;  // this head's channels
          if (a.gn_w) {
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
              const float4 w4 = __ldg(reinterpret_cast<const float4*>(a.gn_w + ch + u));
              x[u] *= w4.x, x[u + 1] *= w4.y, x[u + 2] *= w4.z, x[u + 3] *= w4.w;
            }
          }
          if (a.gn_b) {
#pragma unroll
            for (int u = 0; u < 32; u += 4) {
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(a.gn_b + ch + u));
              x[u] += b4.x, x[u + 1] += b4.y, x[u + 2] += b4.z, x[u + 3] += b4.w;
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) x[u] = yf * __uint_as_float(o[u]);
        }
        if (r < C) store_row32_sw128(ystage, y_box, (uint32_t)r, (uint32_t)c0, x);
      }
      tc_fence_before();
      mbar_arrive(&ofree[ob]);
      fence_proxy_async_smem();
      mbar_arrive(&ystaged[s]);  // the producer stores it
      if (t == 0) RET_TRACE_STAMP(cta_id, it, 7);
      (void)row_lo;
      return true;
    };
    if (nck > 0 && zeta_step(0)) {
      for (int it = 0; it < nck; ++it) {
        if (it + 1 < nck && !zeta_step(it + 1)) break;
        if (!y_step(it)) break;
      }
    }
  } else if (warp >= kWarpSBase) {
    // ---------------------------------------------------- S group (4 warps)
    // TMEM lane v = this thread's dv column of the state S^T.  Keeps the fp32
    // state, its bf16 copy Sb for MMA4 and the gamma^l rescale for MMA5.  In the
    // rescaled form the copy is of the rescaled state.
    const uint32_t v_loc = threadIdx.x - kWarpSBase * 32;
    const uint32_t lane_off = (uint32_t)((warp - kWarpSBase) * 32) << 16;
    const int v = vt * kCW_DVT + (int)v_loc;
    const size_t dkdv = (size_t)DK * a.dv;
    const float g0 = pw[l_first];
    float rho = cw_rho_first(rescaled, g0);
    {
      // the segment states come from the launches before this one on the
      // stream, which may still be running (programmatic dependent launch)
      if (a.n_seg > 1) griddep_wait();
      const bool tr = REV && a.n_seg > 1 && a.seg_state == nullptr && a.seg_tr != nullptr;
      const float* src = (a.n_seg > 1) ? (a.seg_state ? a.seg_state + ((size_t)bh * a.n_seg + seg) * dkdv : nullptr)
                                       : (a.state_in ? a.state_in + (size_t)bh * dkdv : nullptr);
      // transposed source: row v of the [dv][dk] state, contiguous in d
      const float* src_tr = nullptr;
      if (tr) {
        const int slot = (seg == a.n_seg - 1) ? a.seg_tr_nseg - 1 : a.seg_tr_step * (seg + 1) - 1;
        if (RET_BC(slot >= 0 && slot < a.seg_tr_nseg && v < a.dv, 108))
          src_tr = a.seg_tr + ((size_t)bh * a.seg_tr_nseg + slot) * dkdv + (size_t)v * DK;
      }
      // rescaled: U = S_in (or gamma^l0 S_in when rho was reset), Sb = bf16(U);
      // direct: TMEM holds gamma^l0 S_in, Sb = S_in
      const float gu = (rho == 1.f) ? g0 : 1.f;
      const float gc = rescaled ? gu : 1.f;
      for (int d0 = 0; d0 < DK; d0 += 32) {
        float x[32];
        uint32_t w[32];
        if (tr) {
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            const float4 f4 = src_tr ? *reinterpret_cast<const float4*>(src_tr + d0 + u) : make_float4(0.f, 0.f, 0.f, 0.f);
            x[u] = f4.x, x[u + 1] = f4.y, x[u + 2] = f4.z, x[u + 3] = f4.w;
          }
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u)
            x[u] = (src && RET_BC(d0 + u < DK && v < a.dv, 104)) ? src[(size_t)(d0 + u) * a.dv + v] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const float sv = x[u];
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
      if (v_loc == 0) RET_TRACE_STAMP(cta_id, 255, 2);  // trace: initial state in place
    }
    for (int it = 0; it < nck; ++it) {
      // MMA5 (state update) and MMA4 (last reader of Sb) are both done
      if (!mbar_wait(ocross, it & 1, abort_flag, a.lim)) break;
      if (v_loc == 0) RET_TRACE_STAMP(cta_id, it, 10);
      tc_fence_after();
      const int t0 = blk_t0(it);
      if (it < nck - 1) {
        const float gn = pw[blk_len(it + 1)];
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
        if (v_loc == 0) RET_TRACE_STAMP(cta_id, it, 8);
      } else if (a.state_out && seg == (REV ? 0 : a.n_seg - 1)) {
        float* so = a.state_out + (size_t)bh * dkdv;
        for (int d0 = 0; d0 < DK; d0 += 32) {
          uint32_t sr[32];
          tmem_ld32(tm + lane_off + TM_S + d0, sr);
          tmem_ld_wait();
          if (!RET_BC(d0 + 32 <= DK && v < a.dv, 103)) continue;
#pragma unroll
          for (int u = 0; u < 32; ++u) so[(size_t)(d0 + u) * a.dv + v] = rho * __uint_as_float(sr[u]);
        }
      }
    }
  } else {
    // -------------------------------------------------- P/O group (4 warps)
    // TMEM lane r = row r of P and O (token t0 + r of the block).  P -> P~ for
    // MMA3 (and xi on O in the direct form); y is read out by the V group.
    const int r = (int)threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int row_lo = warp * 32;  // rows of this warp: [row_lo, row_lo + 32)
    for (int it = 0; it < nck; ++it) {
      const int t0 = blk_t0(it);
      const int l = min(C, a.L - t0);
      if (!mbar_wait(pfull, it & 1, abort_flag, a.lim)) break;
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 12);
      (void)RET_BC(l >= 1 && l <= C && t0 >= 0 && t0 < a.L, 107);
      tc_fence_after();
      // P -> P~ in place (two bf16 per column).  Rows past the block end read
      // zero Q rows and columns past it zero K rows, so P is already 0 there.
      // Rescaled form: P~ = P on and below the diagonal (decay lives in zeta V
      // and the row factor applied at the end).  Direct form: P~ = P gamma^(r-j).
      const uint32_t tp = tm + lane_off + TM_P;
      for (int j0 = 0; j0 < C; j0 += 32) {
        uint32_t pr[32];
        tmem_ld32(tp + j0, pr);
        tmem_ld_wait();
        uint32_t w[16];
        if (REV ? j0 + 32 <= row_lo : j0 >= row_lo + 32) {
#pragma unroll
          for (int u = 0; u < 16; ++u) w[u] = 0u;
        } else if (rescaled) {
          if ((REV ? j0 >= row_lo + 31 : j0 + 31 <= row_lo)) {
#pragma unroll
            for (int u = 0; u < 32; u += 2) w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]), __uint_as_float(pr[u + 1]));
          } else {
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              const int j = j0 + u;
              w[u / 2] = pack_bf16x2((REV ? (j >= r && j < C) : j <= r) ? __uint_as_float(pr[u]) : 0.f,
                                     (REV ? (j + 1 >= r && j + 1 < C) : j + 1 <= r) ? __uint_as_float(pr[u + 1]) : 0.f);
            }
          }
        } else if ((REV ? j0 >= row_lo + 31 : j0 + 31 <= row_lo)) {
          // whole 32x32 block below the diagonal: gamma^(r-j) = gamma^(r-j0-31) * gamma^(31-u)
          const float ar = pw[REV ? j0 - r : r - j0 - 31];
#pragma unroll
          for (int u = 0; u < 32; u += 2)
            w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * ar * pw[REV ? u : 31 - u],
                                   __uint_as_float(pr[u + 1]) * ar * pw[REV ? u + 1 : 30 - u]);
        } else {
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            const int j = j0 + u;
            const float f0 = (REV ? (j >= r && j < C) : j <= r) ? pw[REV ? j - r : r - j] : 0.f;
            const float f1 = (REV ? (j + 1 >= r && j + 1 < C) : j + 1 <= r) ? pw[REV ? j + 1 - r : r - j - 1] : 0.f;
            w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * f0, __uint_as_float(pr[u + 1]) * f1);
          }
        }
        // When C % 32 == 16 the last piece also covers 16 columns past C; their
        // packed results land at columns >= C/2, which MMA3 never reads.
        tmem_st16(tp + j0 / 2, w);
      }
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 5);
      if (!rescaled) {
        // O *= xi_r = gamma^(r+1) once MMA4 wrote Q S_prev into this block's O buffer
        if (!mbar_wait(ocross, it & 1, abort_flag, a.lim)) break;
        tc_fence_after();
        const float xi = pw[REV ? max(l - r, 0) : r + 1];
        const uint32_t t_o = tm + lane_off + TM_O + 128u * (uint32_t)(it & 1);
        for (int c0 = 0; c0 < kCW_DVT; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(t_o + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * xi);
          tmem_st32(t_o + c0, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(pready);
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 6);
    }
  }
  if (threadIdx.x == 0) bulk_wait_all();  // no store is left in flight (the producer waited for its own)
  if (threadIdx.x == 0) RET_TRACE_STAMP(cta_id, 255, 4);  // trace: end of the roles
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tm, kTmemCols);
  }
}

// ------------------------------------------------------------------------
// dk = 256: one stage, with the scores and the cross-block term fused into a
// single N = C + 128 MMA per K step:  [P | X] = Q [K ; Sb]^T, where the bf16
// state copy Sb sits in shared memory right after the K rows of each 64-column
// box and X (the cross-block term, then the whole output O) sits in TMEM right
// after P.  Q is read once per block and the wide instruction keeps the tensor
// core near its peak rate; TMEM holds S^T [0, 256) and [P | X] [256, 512).
// Order per block: MMA14 ([P | X]; frees Q), MMA5 (state update; frees K),
// MMA3 (X += P~ V; frees V).
struct Cw256Smem {
  uint32_t q, ks, v, misc, total, ks_box;
};

__host__ __device__ inline Cw256Smem cw256_smem_plan(int C) {
  Cw256Smem s;
  s.ks_box = (uint32_t)(C + 128) * 128u;  // K rows 0..C-1, then Sb rows (dv columns 0..127)
  s.q = 0;
  s.ks = 4u * 16384u;
  s.v = s.ks + 4u * s.ks_box;
  s.misc = s.v + 2u * (uint32_t)C * 128u;
  s.total = s.misc + kMiscBytes + kSmemAlign;
  return s;
}

template <bool REV>
__global__ void __launch_bounds__(kCW_MainThreads, 1)
chunkwise_tc256_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, const CwArgs a,
                       const __grid_constant__ CwDecay dec) {
  constexpr int DK = 256;
  constexpr uint32_t kTmemCols = 512, TM_S = 0, TM_P = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem(smem_raw);
  const int C = a.C;
  const uint32_t TM_X = TM_P + (uint32_t)C;
  const Cw256Smem sp = cw256_smem_plan(C);
  uint8_t* sQ = base + sp.q;
  uint8_t* sKS = base + sp.ks;
  uint8_t* sV = base + sp.v;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + sp.misc);
  uint64_t* fullQ = bars + 0;
  uint64_t* fullK = bars + 1;
  uint64_t* fullV = bars + 2;
  uint64_t* emptyQ = bars + 3;     // MMA14 done
  uint64_t* emptyK = bars + 4;     // MMA5 done
  uint64_t* emptyV = bars + 5;     // MMA3 done
  uint64_t* zready = bars + 6;     // V group: zeta applied (to V, or to K in the direct form)
  uint64_t* pxfull = bars + 7;     // MMA14 done -> P/O group, V group (direct form)
  uint64_t* pready = bars + 8;     // P/O group: P~ (and xi X) written -> MMA3
  uint64_t* mma5done = bars + 9;   // MMA5 done -> S group
  uint64_t* sready = bars + 10;    // S group: Sb + rescaled state written -> MMA14, MMA5
  uint64_t* mma3done = bars + 11;  // MMA3 done -> P/O group (y)
  uint64_t* ofree = bars + 12;     // P/O group: X read out -> MMA14 of the next block
  uint64_t* fin = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14) + 1;
  float* pw = reinterpret_cast<float*>(bars + 16);  // gamma^0 .. gamma^128

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vt = blockIdx.x, bh = blockIdx.y, seg = blockIdx.z;
  const float l2g = dec.l2g[bh % a.H];
  const bool rescaled = (float)(C - 1) * l2g >= -64.f;
  const int n_total = (a.L + C - 1) / C;
  const int c_begin = seg * a.seg_chunks;
  const int c_end = min(c_begin + a.seg_chunks, n_total);
  const int nck = max(c_end - c_begin, 0);
  // Step it of the walk takes block blk_idx(it): forward from the segment's
  // first block, REV (the anti-causal sum) from its last block down.
  auto blk_idx = [&](int it) { return REV ? c_end - 1 - it : c_begin + it; };
  auto blk_t0 = [&](int it) { return blk_idx(it) * C; };
  auto blk_len = [&](int it) { return min(C, a.L - blk_t0(it)); };
  const int l_first = nck > 0 ? blk_len(0) : 0;
  const int cta_id = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  (void)cta_id;
  RET_TRACE_INIT();

  if (threadIdx.x == 0) {
    for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
    mbar_init(zready, 256);  // S and V groups each scale half of the tile
    mbar_init(pxfull, 1);
    mbar_init(pready, 128);
    mbar_init(mma5done, 1);
    mbar_init(sready, 256);  // S group and V group each rescale half of dk
    mbar_init(mma3done, 1);
    mbar_init(ofree, 128);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int n = threadIdx.x; n <= 128; n += kCW_MainThreads) pw[n] = n == 0 ? 1.f : exp2f((float)n * l2g);
  if (C < 128) {  // rows C..127 of every Q box are read by the M = 128 MMA: keep them zero
    const uint32_t rows16 = (128u - (uint32_t)C) * 8u;
    for (uint32_t e = threadIdx.x; e < 4u * rows16; e += kCW_MainThreads) {
      const uint32_t b = e / rows16, o = e % rows16;
      *reinterpret_cast<uint4*>(sQ + b * 16384u + (uint32_t)C * 128u + o * 16u) = make_uint4(0, 0, 0, 0);
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
        const int t0 = blk_t0(it);
        if (it >= 1 && !mbar_wait(emptyQ, par, abort_flag, a.lim)) break;
        mbar_arrive_expect_tx(fullQ, qk_bytes);
        for (int b = 0; b < 4; ++b) tma_load_3d(sQ + b * 16384, &mapQ, fullQ, b * 64, t0, bh);
        if (it >= 1 && !mbar_wait(emptyK, par, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, it, 0);
        if (blk_idx(it) != a.debug_drop_block) {  // fault injection: a load that never lands
          mbar_arrive_expect_tx(fullK, qk_bytes);
          for (int b = 0; b < 4; ++b) tma_load_3d(sKS + b * sp.ks_box, &mapK, fullK, b * 64, t0, bh);
        }
        if (it >= 1 && !mbar_wait(emptyV, par, abort_flag, a.lim)) break;
        mbar_arrive_expect_tx(fullV, v_bytes);
        for (int b = 0; b < 2; ++b) tma_load_3d(sV + b * C * 128, &mapV, fullV, vt * kCW_DVT + b * 64, t0, bh);
        issued = it + 1;
        if (it + 1 < nck) {  // next block's tiles into L2 while this one runs
          const int tp = blk_t0(it + 1);
          for (int b = 0; b < 4; ++b) {
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
      const uint32_t id14 = idesc_bf16(128, C + 128, false, false);
      const uint32_t id5 = idesc_bf16(128, DK, true, true);
      const uint32_t id3 = idesc_bf16(128, kCW_DVT, false, true);
      const uint32_t aQ = smem_u32(sQ), aKS = smem_u32(sKS), aV = smem_u32(sV);
      for (int it = 0; it < nck; ++it) {
        const uint32_t par = it & 1;
        if (!mbar_wait4(fullQ, par, fullK, par, sready, par, ofree, par, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, it, 1);
        tc_fence_after();
        // MMA14: [P | X] = Q [K ; Sb]^T
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aQ + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(aKS + (kk / 4) * sp.ks_box + (kk % 4) * 32, 16, 1024);
          mma_ss(tm + TM_P, ad, bd, id14, kk > 0);
        }
        mma_commit(pxfull);
        mma_commit(emptyQ);
        RET_TRACE_STAMP(cta_id, it, 12);
        // MMA5: S^T += (zeta V)^T K  (rescaled: zeta on V; direct: zeta on K)
        if (!mbar_wait(zready, par, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, it, 2);
        tc_fence_after();
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aV + kk * 2048, C * 128, 1024);
          const uint64_t bd = sdesc_sw128(aKS + kk * 2048, sp.ks_box, 1024);
          mma_ss(tm + TM_S, ad, bd, id5, 1);
        }
        mma_commit(mma5done);
        mma_commit(emptyK);
        RET_TRACE_STAMP(cta_id, it, 13);
        // MMA3: X += P~ V
        if (!mbar_wait(pready, par, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, it, 4);
        tc_fence_after();
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(aV + kk * 2048, C * 128, 1024);
          mma_ts(tm + TM_X, tm + TM_P + kk * 8, bd, id3, 1);
        }
        mma_commit(mma3done);
        mma_commit(emptyV);
        RET_TRACE_STAMP(cta_id, it, 14);
      }
      mma_commit(fin);
      mbar_drain(fin, 0, a.lim);
    }
  } else if (warp >= kWarpSBase) {
    // ------------------------------------------ S group and V group (8 warps)
    // Both keep the state: lane v owns dv column v of S^T; the S group the dk
    // columns [0, 128), the V group [128, 256).  The state copy Sb sits in rows
    // C..C+127 of each KS box.  The V group also applies zeta_j = gamma^(l-1-j)
    // (0 past the block end) to row j of V (rescaled form, as soon as V lands)
    // or of K (direct form, once MMA14 has read the unscaled K).
    const bool vgrp = warp >= kWarpZBase;
    const int gbase = vgrp ? kWarpZBase : kWarpSBase;
    const uint32_t v_loc = threadIdx.x - gbase * 32;
    const uint32_t lane_off = (uint32_t)((warp - gbase) * 32) << 16;
    const int half = vgrp ? 1 : 0;
    const int d_lo = 128 * half;
    const int v = vt * kCW_DVT + (int)v_loc;
    const size_t dkdv = (size_t)DK * a.dv;
    uint8_t* sSb = sKS + (uint32_t)C * 128u;  // first Sb row of box 0; box stride ks_box
    const float g0 = pw[l_first];
    float rho = cw_rho_first(rescaled, g0);
    {
      if (a.n_seg > 1) griddep_wait();  // segment states from the launches before (see above)
      const float* src = (a.n_seg > 1) ? a.seg_state + ((size_t)bh * a.n_seg + seg) * dkdv
                                       : (a.state_in ? a.state_in + (size_t)bh * dkdv : nullptr);
      // TMEM starts as gu S_in: rescaled, U = S_in (or gamma^l0 S_in when rho
      // was reset); direct, the decayed state gamma^l0 S_in.  Sb = bf16(U) in
      // the rescaled form, S_in in the direct form.
      const float gu = (rho == 1.f) ? g0 : 1.f;
      const float gc = rescaled ? gu : 1.f;
      for (int d0 = d_lo; d0 < d_lo + 128; d0 += 32) {
        float x[32];
        uint32_t w[32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const float sv = (src && RET_BC(d0 + u < DK && v < a.dv, 104)) ? src[(size_t)(d0 + u) * a.dv + v] : 0.f;
          x[u] = gc * sv;
          w[u] = __float_as_uint(gu * sv);
        }
        store_row32_sw128(sSb, sp.ks_box, v_loc, d0, x);
        tmem_st32(tm + lane_off + TM_S + d0, w);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(sready);
    }
    for (int it = 0; it < nck; ++it) {
      const uint32_t par = it & 1;
      const int t0 = blk_t0(it);
      {
        // zeta (rescaled: zeta / rho) on row v_loc of V (rescaled form, as soon
        // as V lands) or of K (direct form, once MMA14 has read it); the S group
        // takes the first half of the row's 64-column boxes, the V group the rest.
        if (!mbar_wait(fullV, par, abort_flag, a.lim)) break;
        if (v_loc == 0 && vgrp) RET_TRACE_STAMP(cta_id, it, 9);
        if (!rescaled) {
          if (!mbar_wait(fullK, par, abort_flag, a.lim)) break;
          if (!mbar_wait(pxfull, par, abort_flag, a.lim)) break;
        }
        const int l = min(C, a.L - t0);
        if ((int)v_loc < C) {
          const float zeta = ((int)v_loc < l) ? pw[REV ? (int)v_loc : l - 1 - (int)v_loc] : 0.f;
          if (rescaled) {
            scale_row_sw128(sV + half * C * 128, v_loc, zeta * __frcp_rn(rho));
          } else {
            for (int b = 2 * half; b < 2 * half + 2; ++b) scale_row_sw128(sKS + b * sp.ks_box, v_loc, zeta);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(zready);
        if (v_loc == 0 && vgrp) RET_TRACE_STAMP(cta_id, it, 3);
      }
      // MMA5 done; MMA14 (the reader of the old Sb) ran before it
      if (!mbar_wait(mma5done, par, abort_flag, a.lim)) break;
      if (v_loc == 0 && !vgrp) RET_TRACE_STAMP(cta_id, it, 5);
      tc_fence_after();
      if (it < nck - 1) {
        const float gn = pw[blk_len(it + 1)];
        // direct form: decay the state in TMEM, Sb = S.  Rescaled form: Sb = U,
        // and U is multiplied through only when rho is reset.
        const float rho_n = rescaled ? cw_rho_next(rho, gn) : 1.f;
        const bool write_back = !rescaled || rho_n == 1.f;
        const float mult = rescaled ? gn * rho : gn;
        for (int d0 = d_lo; d0 < d_lo + 128; d0 += 32) {
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
          store_row32_sw128(sSb, sp.ks_box, v_loc, d0, x);
        }
        rho = rho_n;
        if (write_back) tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(sready);
        if (v_loc == 0 && !vgrp) RET_TRACE_STAMP(cta_id, it, 8);
      } else if (a.state_out && seg == (REV ? 0 : a.n_seg - 1)) {
        float* so = a.state_out + (size_t)bh * dkdv;
        for (int d0 = d_lo; d0 < d_lo + 128; d0 += 32) {
          uint32_t sr[32];
          tmem_ld32(tm + lane_off + TM_S + d0, sr);
          tmem_ld_wait();
          if (!RET_BC(d0 + 32 <= DK && v < a.dv, 103)) continue;
#pragma unroll
          for (int u = 0; u < 32; ++u) so[(size_t)(d0 + u) * a.dv + v] = rho * __uint_as_float(sr[u]);
        }
      }
    }
  } else {
    // -------------------------------------------------- P/O group (4 warps)
    const int r = (int)threadIdx.x;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int row_lo = warp * 32;
    float rho = cw_rho_first(rescaled, pw[l_first]);
    mbar_arrive(ofree);  // X starts free
    for (int it = 0; it < nck; ++it) {
      const uint32_t par = it & 1;
      const int t0 = blk_t0(it);
      const int l = min(C, a.L - t0);
      if (!mbar_wait(pxfull, par, abort_flag, a.lim)) break;
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 10);
      (void)RET_BC(l >= 1 && l <= C && t0 >= 0 && t0 < a.L, 207);
      tc_fence_after();
      // P -> P~ in place (see the main kernel for the two forms)
      const uint32_t tp = tm + lane_off + TM_P;
      for (int j0 = 0; j0 < C; j0 += 32) {
        uint32_t pr[32];
        tmem_ld32(tp + j0, pr);
        tmem_ld_wait();
        uint32_t w[16];
        if (REV ? j0 + 32 <= row_lo : j0 >= row_lo + 32) {
#pragma unroll
          for (int u = 0; u < 16; ++u) w[u] = 0u;
        } else if (rescaled) {
          if ((REV ? j0 >= row_lo + 31 : j0 + 31 <= row_lo)) {
#pragma unroll
            for (int u = 0; u < 32; u += 2) w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]), __uint_as_float(pr[u + 1]));
          } else {
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              const int j = j0 + u;
              w[u / 2] = pack_bf16x2((REV ? (j >= r && j < C) : j <= r) ? __uint_as_float(pr[u]) : 0.f,
                                     (REV ? (j + 1 >= r && j + 1 < C) : j + 1 <= r) ? __uint_as_float(pr[u + 1]) : 0.f);
            }
          }
        } else if ((REV ? j0 >= row_lo + 31 : j0 + 31 <= row_lo)) {
          const float ar = pw[REV ? j0 - r : r - j0 - 31];
#pragma unroll
          for (int u = 0; u < 32; u += 2)
            w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * ar * pw[REV ? u : 31 - u],
                                   __uint_as_float(pr[u + 1]) * ar * pw[REV ? u + 1 : 30 - u]);
        } else {
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            const int j = j0 + u;
            const float f0 = (REV ? (j >= r && j < C) : j <= r) ? pw[REV ? j - r : r - j] : 0.f;
            const float f1 = (REV ? (j + 1 >= r && j + 1 < C) : j + 1 <= r) ? pw[REV ? j + 1 - r : r - j - 1] : 0.f;
            w[u / 2] = pack_bf16x2(__uint_as_float(pr[u]) * f0, __uint_as_float(pr[u + 1]) * f1);
          }
        }
        // For C % 32 == 16 the last piece reads 16 columns past P (the start of
        // X) and writes packed results below column C/2 + 8 < C: never into X,
        // never read by MMA3.
        tmem_st16(tp + j0 / 2, w);
      }
      if (!rescaled) {
        // X *= xi_r = gamma^(r+1): X holds Q S_prev from MMA14
        const float xi = pw[REV ? max(l - r, 0) : r + 1];
        for (int c0 = 0; c0 < kCW_DVT; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tm + lane_off + TM_X + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * xi);
          tmem_st32(tm + lane_off + TM_X + c0, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(pready);
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 6);
      // y = (gamma^(r+1-l) in the rescaled form) X, once MMA3 is done
      if (!mbar_wait(mma3done, par, abort_flag, a.lim)) break;
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 11);
      tc_fence_after();
      {
        // X -> registers as bf16 pairs, release X to the next block's MMA14,
        // then the global stores.
        const float yf = rescaled ? exp2f((float)(REV ? -r : r + 1 - l) * l2g) * rho : 1.f;
        __nv_bfloat16* wrow0 = a.y + ((size_t)bh * a.L + t0 + row_lo) * a.dv + vt * kCW_DVT;
        uint32_t yb[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tm + lane_off + TM_X + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; ++u)
            yb[c][u] = pack_bf16x2(yf * __uint_as_float(o[2 * u]), yf * __uint_as_float(o[2 * u + 1]));
        }
        tc_fence_before();
        mbar_arrive(ofree);
        if (RET_BC(t0 + l <= a.L && vt * kCW_DVT + 128 <= a.dv, 202)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) store_rows_packed_quad(wrow0 + 32 * c, (size_t)a.dv, lane, yb[c], l - row_lo);
        }
      }
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 7);
      if (it + 1 < nck && rescaled) rho = cw_rho_next(rho, pw[blk_len(it + 1)]);
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

// ------------------------------------------------------------------------
// Segment sums for the sequence split: for segment g of one (b, h) and one
// 128-column dv slice,  D_g^T = sum_{t in g} gamma^(e_g - t) v_t^T k_t  with e_g
// the segment's last token, written (as [dk][dv], like a state) to slot g+1 of
// the workspace [BH][n_seg][dk][dv].  Rows of K (DK <= 128) or of V (DK = 256)
// are scaled by the decay to the segment end in shared memory, then
// accumulated by tcgen05 into TMEM.
// REV (the anti-causal sum): the sum of segment g = 1..n_seg-1 decays to the
// segment's FIRST token s_g, D_g^T = sum_{t in g} gamma^(t - s_g) v_t^T k_t,
// and goes to slot g-1.
template <int DK, bool REV>
__global__ void __launch_bounds__(kCW_Threads)
chunk_state_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                   const CwArgs a, const __grid_constant__ CwDecay dec, float* ws) {
  constexpr uint32_t kTmemCols = DK;  // 64, 128 or 256: powers of two >= 32
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_smem(smem_raw);
  const int C = a.C, NS = a.nstages;
  const uint32_t k_stage = (uint32_t)(DK / 64) * C * 128, v_stage = 2u * C * 128;
  uint8_t* sK = base;
  uint8_t* sV = base + NS * k_stage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + NS * (k_stage + v_stage));
  uint64_t* full = bars;        // [4]
  uint64_t* empty = bars + 4;   // [4]
  uint64_t* kready = bars + 8;  // [4] epilogue scaled the K or V rows -> MMA
  uint64_t* done = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 13) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vt = blockIdx.x, bh = blockIdx.y;
  const int seg = REV ? (int)blockIdx.z + 1 : (int)blockIdx.z;  // forward: seg < n_seg - 1; REV: seg >= 1
  const float l2g = dec.l2g[bh % a.H];
  const int n_total = (a.L + C - 1) / C;
  const int c_begin = seg * a.seg_chunks;
  const int c_end = min(c_begin + a.seg_chunks, n_total);
  const int nck = max(c_end - c_begin, 0);
  const int seg_last = min(c_end * C, a.L) - 1;  // e_g
  const int seg_first = c_begin * C;              // s_g
  const int cta_id = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  (void)cta_id;
  RET_TRACE_INIT();

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&kready[i], 128);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tmem_slot;

  if (warp == 4) {
    if (lane == 0 && nck > 0) {
      const uint32_t bytes = (uint32_t)(DK + kCW_DVT) * C * 2u;
      int issued = 0;
      for (int it = 0; it < nck; ++it) {
        const int s = it % NS;
        if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1, abort_flag, a.lim)) break;
        const int t0 = (c_begin + it) * C;
        RET_TRACE_STAMP(cta_id, it, 0);
        mbar_arrive_expect_tx(&full[s], bytes);
        for (int b = 0; b < DK / 64; ++b)
          tma_load_3d(sK + s * k_stage + b * C * 128, &mapK, &full[s], b * 64, t0, bh);
        for (int b = 0; b < 2; ++b)
          tma_load_3d(sV + s * v_stage + b * C * 128, &mapV, &full[s], vt * kCW_DVT + b * 64, t0, bh);
        issued = it + 1;
      }
      for (int it = max(0, issued - NS); it < issued; ++it) mbar_drain(&full[it % NS], (it / NS) & 1, a.lim);
    }
  } else if (warp == 5) {
    if (lane == 0 && nck > 0) {
      const uint32_t id5 = idesc_bf16(128, DK, true, true);
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
      for (int it = 0; it < nck; ++it) {
        const int s = it % NS;
        if (!mbar_wait(&full[s], (it / NS) & 1, abort_flag, a.lim)) break;
        if (!mbar_wait(&kready[s], (it / NS) & 1, abort_flag, a.lim)) break;
        RET_TRACE_STAMP(cta_id, it, 1);
        tc_fence_after();
        for (int kk = 0; kk < C / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aV + s * v_stage + kk * 2048, C * 128, 1024);
          const uint64_t bd = sdesc_sw128(aK + s * k_stage + kk * 2048, C * 128, 1024);
          mma_ss(tm, ad, bd, id5, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        RET_TRACE_STAMP(cta_id, it, 4);
      }
      mma_commit(done);
    }
  } else {
    const uint32_t r = threadIdx.x;
    bool ok = true;
    for (int it = 0; it < nck; ++it) {
      const int s = it % NS;
      if (!mbar_wait(&full[s], (it / NS) & 1, abort_flag, a.lim)) { ok = false; break; }
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 2);
      // Row j of the narrower operand times gamma^(e_g - t).  DK <= 128: rows
      // of K, one row per thread.  DK = 256: rows of V (half the bytes of
      // K's): thread r takes 64-column box (r & 1) of row (r >> 1), all 8
      // loads first, one factor per thread.
      if constexpr (DK <= kCW_DVT) {
        for (uint32_t j = r; j < (uint32_t)C; j += 128) {  // rows j and j + 128 (blocks up to 256)
          const int t = (c_begin + it) * C + (int)j;
          const int ex = REV ? t - seg_first : seg_last - t;
          const float f = (t <= seg_last) ? (ex == 0 ? 1.f : exp2f((float)ex * l2g)) : 0.f;
          for (int b = 0; b < DK / 64; ++b) scale_row_sw128(sK + s * k_stage + b * C * 128, j, f);
        }
      } else {
        uint8_t* vs = sV + s * v_stage;
        for (uint32_t pr = r; pr < 2u * (uint32_t)C; pr += 128) {
          const uint32_t j = pr >> 1;
          const int t = (c_begin + it) * C + (int)j;
          const int ex = REV ? t - seg_first : seg_last - t;
          const float f = (t <= seg_last) ? (ex == 0 ? 1.f : exp2f((float)ex * l2g)) : 0.f;
          scale_row_sw128(vs + (pr & 1u) * (uint32_t)C * 128u, j, f);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&kready[s]);
      if (r == 0) RET_TRACE_STAMP(cta_id, it, 3);
    }
    if (ok && nck > 0 && mbar_wait(done, 0, abort_flag, a.lim)) {
      tc_fence_after();
      const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
      const size_t dkdv = (size_t)DK * a.dv;
      const int slot = REV ? seg - 1 : seg + 1;
      float* dst = ws + ((size_t)bh * a.n_seg + slot) * dkdv;
      const int v = vt * kCW_DVT + (int)r;
      for (int d0 = 0; d0 < DK && RET_BC(slot >= 0 && slot < a.n_seg && v < a.dv, 401); d0 += 32) {
        uint32_t sr[32];
        tmem_ld32(tm + lane_off + d0, sr);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 32; ++u) dst[(size_t)(d0 + u) * a.dv + v] = __uint_as_float(sr[u]);
      }
    }
  }
  // The scan (or fold) that consumes the segment sums may be launched now; it
  // waits for this grid's completion before it reads them.
  if (threadIdx.x == 0) griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    if (lane == 0 && nck > 0) {
      // no MMA may still be running when TMEM is released
      mbar_drain(done, 0, a.lim);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tm, kTmemCols);
  }
}

// Scan over segments, element-wise on the state: slot 0 <- S_in, and for
// g = 1..n_seg-1, slot g <- gamma^len * slot(g-1) + D_(g-1) (D_(g-1) was stored in
// slot g by chunk_state_kernel).  len = tokens per segment (all but the last
// segment are full).
// REV: slot n_seg-1 <- S_in (the state after the sequence), and for
// g = n_seg-2..0, slot g <- gamma^len(g+1) * slot(g+1) + D_(g+1) (stored in
// slot g); the last segment has last_len tokens.
template <bool REV>
__global__ void state_scan_kernel(const float* __restrict__ state_in, float* __restrict__ ws,
                                  int BH, int H, int dkdv, int n_seg, int seg_len, int last_len,
                                  const __grid_constant__ CwDecay dec) {
  // One element per thread; the segment sums are loaded eight at a time
  // ahead of the dependent multiply-adds, so the chain waits on arithmetic,
  // not on one memory round trip per segment.
  griddep_wait();  // the segment sums of chunk_state_kernel
  const size_t total = (size_t)BH * dkdv;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int bh = (int)(e / dkdv);
    const size_t off = e % dkdv;
    const float gl = exp2f((float)seg_len * dec.l2g[bh % H]);
    float S = state_in ? state_in[e] : 0.f;
    float* slot = ws + (size_t)bh * n_seg * dkdv + off;
    if (!REV) {
      slot[0] = S;
      for (int g0 = 1; g0 < n_seg; g0 += 8) {
        float d[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) d[u] = (g0 + u < n_seg) ? slot[(size_t)(g0 + u) * dkdv] : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (g0 + u < n_seg) {
            S = fmaf(gl, S, d[u]);
            slot[(size_t)(g0 + u) * dkdv] = S;
          }
      }
    } else {
      const float gl_last = exp2f((float)last_len * dec.l2g[bh % H]);
      slot[(size_t)(n_seg - 1) * dkdv] = S;
      for (int g0 = n_seg - 2; g0 >= 0; g0 -= 8) {
        float d[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) d[u] = (g0 - u >= 0) ? slot[(size_t)(g0 - u) * dkdv] : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (g0 - u >= 0) {
            S = fmaf(g0 - u + 1 == n_seg - 1 ? gl_last : gl, S, d[u]);
            slot[(size_t)(g0 - u) * dkdv] = S;
          }
      }
    }
  }
  // the main kernel, launched behind this one, waits for its completion
  if (threadIdx.x == 0) griddep_launch_dependents();
}

}  // namespace ret
