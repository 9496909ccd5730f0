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
