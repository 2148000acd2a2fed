// backward.cuh -- pieces of the backward pass of the parallel form.
//
// With y_n = sum_{m<=n} gamma^(n-m) (q_n . k_m) v_m (page "Retentive Networks
// -- Microsoft ...", section "Il meccanismo: Multi-Scale Retention") and an
// upstream gradient dy, the chain rule gives three sums of the same kind:
//     dq_n = sum_{m<=n} gamma^(n-m) (dy_n . v_m) k_m     = retention(dy, v, k)_n
//     dk_m = sum_{n>=m} gamma^(n-m) (dy_n . v_m) q_n
//     dv_m = sum_{n>=m} gamma^(n-m) (q_n . k_m) dy_n
// The last two run backwards in time: with R the reversal of the sequence
// axis, dk = R(retention(R v, R dy, R q)) and dv = R(retention(R k, R q, R dy)).
// So the backward pass is three launches of the forward parallel kernel plus
// the reversals below.
#pragma once
#include <stdint.h>

namespace ret {

// out[bh][L-1-n][:] = in[bh][n][:] for rows of `row_bytes` bytes, copied in
// units of U (uint4 when row_bytes % 16 == 0, else uint32_t or uint16_t).
template <typename U>
__global__ void __launch_bounds__(256) reverse_rows_kernel(const U* __restrict__ in, U* __restrict__ out,
                                                           long long BH, int L, int units_per_row) {
  const long long total = BH * L * (long long)units_per_row;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / units_per_row;
    const int u = (int)(e % units_per_row);
    const long long bh = row / L;
    const int n = (int)(row % L);
    out[(bh * L + (L - 1 - n)) * units_per_row + u] = in[e];
  }
}

}  // namespace ret
