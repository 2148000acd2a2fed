// state_fold.cuh -- the recurrence between blocks, applied to whole runs of
// tokens at once.
//
// The state after a run of `len` tokens that starts from S is
//     gamma^len S + D,   D = sum_t gamma^(len-1-t) k_t^T v_t
// (unrolling the recurrence S_n = gamma S_(n-1) + k_n^T v_n of the page
// "Retentive Networks -- Microsoft ...", section "Il meccanismo", over the
// run).  D is the run's state from zero.  So the state at the start of run i of
// a sequence cut into runs 0, 1, ... follows from the runs' D alone:
//     S_0 = S_in,   S_(i+1) = gamma^len_i S_i + D_i.
// state_fold_kernel evaluates this fold elementwise over the dk x dv state.
// It joins the per-segment sums of one long call on one GPU, and the
// per-rank sums of a sequence cut across GPUs (each rank folds the parts of
// the ranks before it).
#pragma once
#include <stdint.h>

#include "simt_f32.cuh"  // HeadLog2, decay_pow
#include "tc_common.cuh"  // griddep_wait

namespace ret {

constexpr int kFoldMaxParts = 256;

struct FoldLens {
  int len[kFoldMaxParts];  // tokens in each run
};

// out[bh][e] = fold over parts i < n of (gamma_h^len_i * S + part_i), S starting
// at state_in[bh][e] (or 0).  Part i of row bh sits at
// parts + i * part_stride + bh * bh_stride (floats).  out may alias state_in.
__global__ void __launch_bounds__(256) state_fold_kernel(const float* state_in, const float* __restrict__ parts,
                                                         float* out, long long BH, int H, int dkdv, int n,
                                                         long long part_stride, long long bh_stride,
                                                         const __grid_constant__ HeadLog2 hl,
                                                         const __grid_constant__ FoldLens fl) {
  griddep_wait();  // parts written by the launch before this one (if it was programmatic)
  const long long total = BH * dkdv;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long bh = e / dkdv;
    const int off = (int)(e % dkdv);
    const float l2g = hl.l2g[bh % H];
    float S = state_in ? state_in[e] : 0.f;
    const float* p = parts + bh * bh_stride + off;
    for (int i = 0; i < n; ++i) S = fmaf(decay_pow(l2g, fl.len[i]), S, p[(long long)i * part_stride]);
    out[e] = S;
  }
}

}  // namespace ret
