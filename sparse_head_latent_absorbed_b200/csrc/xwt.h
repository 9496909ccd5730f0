// Weight-streaming GEMM shared by the projections of the attention block:
//   Y[b, n] = sum_k X[b, k] W[n, k]      X bf16 [B, K], W bf16 [N, K] ([out, in])
// computed as fp32 partials of D^T = W X^T (xwt_gemm, in out_proj.cu), to be
// summed and finished by a per-projection kernel.
//
// Work split: row tile m (128 rows of W) and K chunk j (128 columns) form unit
// m * nch + j; persistent CTA c takes units [bnd(c), bnd(c+1)) for each block
// of 128 batch rows.  The part of a row tile one CTA holds ends in an fp32
// partial at part[((m * slots + (c - c_first(m))) * B + b) * 128 + row]; a
// finishing kernel sums slots 0 .. c_last(m) - c_first(m) of tile m in that
// order, so results do not depend on timing.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/shla.h"

namespace shla {

struct XwtSched {
  int tot;    // row tiles x chunks
  int nc;     // CTAs per block of batch rows
  int nch;    // K chunks per row tile
  int slots;  // partial slots per row tile (the most CTAs any tile meets)
  __host__ __device__ int bnd(int c) const { return (int)((long long)c * tot / nc); }
  __host__ __device__ int c_first(int m) const {
    return (int)((((long long)m * nch + 1) * nc + tot - 1) / tot) - 1;
  }
  __host__ __device__ int c_last(int m) const {
    return (int)((((long long)(m + 1) * nch) * nc + tot - 1) / tot) - 1;
  }
};

// acc[0..7] += the partials of outputs nl .. nl + 7 of row tile m, batch row
// b, in slots s0, s0 + step, s0 + 2 step, ... below `used`, added in slot
// order; the loads of kBatch slots are in flight together.
template <int kBatch>
__device__ __forceinline__ void xwt_sum_slots(const float* __restrict__ part, const XwtSched& sch,
                                              int m, int nl, int b, int B, int s0, int step,
                                              int used, float (&acc)[8]) {
#pragma unroll 1
  for (int base = s0; base < used; base += kBatch * step) {
    float4 v[kBatch][2];
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const int s = base + t * step;
      if (s < used) {
        const float4* src =
            reinterpret_cast<const float4*>(part + ((size_t)(m * sch.slots + s) * B + b) * 128 + nl);
        v[t][0] = src[0];
        v[t][1] = src[1];
      }
    }
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      if (base + t * step < used) {
        acc[0] += v[t][0].x;
        acc[1] += v[t][0].y;
        acc[2] += v[t][0].z;
        acc[3] += v[t][0].w;
        acc[4] += v[t][1].x;
        acc[5] += v[t][1].y;
        acc[6] += v[t][1].z;
        acc[7] += v[t][1].w;
      }
    }
  }
}

// CTAs per block of batch rows: min(148, units), the same on every device,
// so the summation order (and with it every result bit) does not depend on
// the device
constexpr int kXwtCtas = 148;

// plan for a [n_out, k_in] weight (n_out % 128 == 0, k_in % 128 == 0)
XwtSched xwt_plan(int n_out, int k_in);

// fp32 partial bytes for B rows under `plan`
size_t xwt_part_bytes(const XwtSched& plan, int n_out, int B);

// enqueue the partials of Y = X W^T; returns MLA_OK or an MLA_ERR_* code.
// pdl: launch with programmatic serialisation after a kernel of the same call
// (the weight must not be written by that kernel; X and part may be).
int xwt_gemm(const void* w, int n_out, int k_in, const void* x, int B, float* part,
             const XwtSched& plan, int32_t* status, cudaStream_t st, bool pdl);

}  // namespace shla
