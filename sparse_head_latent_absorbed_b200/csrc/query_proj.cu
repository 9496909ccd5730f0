// Query path of the attention block ("Query rotary up-projection" page: the
// MLA init and forward excerpts):
//
//   qr    = RMSNorm(x wq_a^T) * w              x bf16 [B, 7168], wq_a [1536, 7168]
//   q     = qr wq_b^T viewed [B, 128, 192]     wq_b [128 * 192, 1536] ([out, in])
//   q_nope = q[..., 0:128],  q_pe = RoPE(q[..., 128:192]) at each row's position
//
// Both projections run on the weight-streaming GEMM of xwt.h; the finishing
// kernels here sum its fp32 partial slots in a fixed order and apply the
// norm (qa_finish) or the split and the rotation (qb_finish).  The RMSNorm
// form and eps follow the cache write's latent norm: y = x / sqrt(mean(x^2) +
// eps) * w, in fp32 on the unrounded projection; qr is rounded to bf16 as the
// second GEMM's operand.  The rotation is the interleaved one the model uses
// for the query's rotary part, with the fp32 (cos, sin) table given as input.
#include <cuda_runtime.h>

#include "common.cuh"
#include "host_util.h"
#include "xwt.h"

namespace shla {
namespace qproj {
constexpr int DIM = 7168;                 // model width
constexpr int QL = 1536;                  // q latent (q_lora_rank)
constexpr int NH = 128, DN = 128, RR = 64;
constexpr int QW = NH * (DN + RR);        // 24576 outputs of wq_b
}  // namespace qproj

// qr[b, :] = bf16(RMSNorm(sum of the slots) * w): one block per row.  Thread
// (g, i) of 4 groups x 192 sums slots g, g + 4, g + 8, ... of outputs
// 8i .. 8i + 7 (four times the loads in flight of one thread per output
// octet); group 0 adds the other groups' sums in group order, so the result
// does not depend on timing.
constexpr int QA_GROUPS = 4;
constexpr int QA_THREADS = 192 * QA_GROUPS;

__global__ void __launch_bounds__(QA_THREADS) qa_finish(const float* __restrict__ part,
                                                        XwtSched sch, int B,
                                                        const __nv_bfloat16* __restrict__ norm_w,
                                                        float eps, __nv_bfloat16* __restrict__ qr) {
  using namespace qproj;
  __shared__ __align__(16) float gsum[QA_GROUPS - 1][QL];
  __shared__ float red[6];
  const int b = blockIdx.x, t = threadIdx.x;
  const int g = t / 192, i = t - g * 192;
  const int n0 = i * 8, m = n0 / 128, nl = n0 % 128;
  const int used = sch.c_last(m) - sch.c_first(m) + 1;
  pdl_trigger();  // the second GEMM may set up and prefetch its weight now
  pdl_wait();     // the partials of the first GEMM
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  xwt_sum_slots<4>(part, sch, m, nl, b, B, g, QA_GROUPS, used, v);
  if (g > 0) {
    float4* dst = reinterpret_cast<float4*>(&gsum[g - 1][n0]);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  __syncthreads();
  if (g == 0) {  // warps 0-5
#pragma unroll
    for (int h = 0; h < QA_GROUPS - 1; ++h) {
      const float4* src = reinterpret_cast<const float4*>(&gsum[h][n0]);
      const float4 a = src[0], c = src[1];
      v[0] += a.x;
      v[1] += a.y;
      v[2] += a.z;
      v[3] += a.w;
      v[4] += c.x;
      v[5] += c.y;
      v[6] += c.z;
      v[7] += c.w;
    }
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) ss += v[k] * v[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((t & 31) == 0) red[t >> 5] = ss;
  }
  __syncthreads();
  if (g != 0) return;
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 6; ++w) tot += red[w];  // fixed order in every thread
  const float inv = rsqrtf(tot / QL + eps);
  const uint4 wv = *reinterpret_cast<const uint4*>(norm_w + n0);
  const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&wv);
  uint4 o;
  uint32_t* op = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 wf = __bfloat1622float2(wp[k]);
    op[k] = pack_bf16x2(v[2 * k] * inv * wf.x, v[2 * k + 1] * inv * wf.y);
  }
  *reinterpret_cast<uint4*>(qr + (size_t)b * QL + n0) = o;
}

// q_nope / q_pe from the slots of wq_b: grid (B, QW / 1024), 128 threads of 8
// consecutive outputs (a thread's 8 never straddle a head or the nope/rope
// boundary).  A row whose position is outside [0, T) gets q_pe = 0 and is
// counted once in status[1].
__global__ void __launch_bounds__(128) qb_finish(const float* __restrict__ part, XwtSched sch,
                                                  int B, const float2* __restrict__ rope, int T,
                                                  const int32_t* __restrict__ pos,
                                                  __nv_bfloat16* __restrict__ q_nope,
                                                  __nv_bfloat16* __restrict__ q_pe,
                                                  int32_t* status) {
  using namespace qproj;
  const int b = blockIdx.x;
  const int n0 = (blockIdx.y * 128 + threadIdx.x) * 8;
  if (n0 >= QW) return;
  const int h = n0 / (DN + RR), e = n0 - h * (DN + RR);
  const int m = n0 / 128, nl = n0 % 128;
  const int used = sch.c_last(m) - sch.c_first(m) + 1;
  pdl_wait();  // the partials of the second GEMM
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  xwt_sum_slots<2>(part, sch, m, nl, b, B, 0, 1, used, v);
  uint4 o;
  uint32_t* op = reinterpret_cast<uint32_t*>(&o);
  if (e < DN) {
#pragma unroll
    for (int i = 0; i < 4; ++i) op[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(q_nope + ((size_t)b * NH + h) * DN + e) = o;
  } else {
    const int r = e - DN;  // first rotary feature of this thread: pairs r/2 .. r/2 + 3
    const int p = pos[b];
    const bool ok = p >= 0 && p < T;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (ok) {
        const float2 cs = rope[(size_t)p * (RR / 2) + r / 2 + i];
        const float x0 = v[2 * i], x1 = v[2 * i + 1];
        op[i] = pack_bf16x2(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);  // (x0 + i x1)(cos + i sin)
      } else {
        op[i] = 0u;
      }
    }
    *reinterpret_cast<uint4*>(q_pe + ((size_t)b * NH + h) * RR + r) = o;
    if (!ok && h == 0 && r == 0 && status) atomicAdd(status + 1, 1);
  }
}

}  // namespace shla

using namespace shla;

// workspace: the larger of the two GEMMs' partial slots, then qr (bf16 [B, 1536])
static size_t qproj_part_bytes(int B) {
  const XwtSched pa = xwt_plan(qproj::QL, qproj::DIM);
  const XwtSched pb = xwt_plan(qproj::QW, qproj::QL);
  const size_t a = xwt_part_bytes(pa, qproj::QL, B), b = xwt_part_bytes(pb, qproj::QW, B);
  return round_up(a > b ? a : b, 256);
}

extern "C" size_t mla_query_proj_workspace_bytes(int B) {
  if (B < 1 || B > 65535) return 0;
  return qproj_part_bytes(B) + round_up((size_t)B * qproj::QL * 2, 256);
}

extern "C" int mla_query_proj(const mla_bf16_t* x, const mla_bf16_t* wq_a,
                              const mla_bf16_t* q_norm_w, float eps, const mla_bf16_t* wq_b,
                              const float* rope, int T, const int32_t* pos, int B,
                              mla_bf16_t* q_nope, mla_bf16_t* q_pe, void* ws, size_t ws_bytes,
                              int32_t* status, void* stream) {
  if (!x || !wq_a || !q_norm_w || !wq_b || !rope || !pos || !q_nope || !q_pe) return MLA_ERR_NULL;
  if (B < 1 || B > 65535 || T < 1 || !(eps >= 0.f)) return MLA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(wq_a) || !aligned16(q_norm_w) || !aligned16(wq_b) ||
      !aligned16(rope) || !aligned16(q_nope) || !aligned16(q_pe))
    return MLA_ERR_ALIGN;
  if (!ws || !aligned256(ws) || ws_bytes < mla_query_proj_workspace_bytes(B))
    return MLA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  cudaStream_t st = as_stream(stream);
  float* part = static_cast<float*>(ws);
  __nv_bfloat16* qr =
      reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + qproj_part_bytes(B));
  const XwtSched pa = xwt_plan(qproj::QL, qproj::DIM);
  // the three kernels after the first are launched with programmatic
  // serialisation: each prepares while its predecessor drains
  if (int e = xwt_gemm(wq_a, qproj::QL, qproj::DIM, x, B, part, pa, status, st, false)) return e;
  if (int e = launch_pdl(qa_finish, dim3(B), dim3(QA_THREADS), 0, st, part, pa, B,
                         reinterpret_cast<const __nv_bfloat16*>(q_norm_w), eps, qr))
    return e;
  const XwtSched pb = xwt_plan(qproj::QW, qproj::QL);
  if (int e = xwt_gemm(wq_b, qproj::QW, qproj::QL, qr, B, part, pb, status, st, true)) return e;
  return launch_pdl(qb_finish, dim3(B, qproj::QW / 1024), dim3(128), 0, st, part, pb, B,
                    reinterpret_cast<const float2*>(rope), T, pos,
                    reinterpret_cast<__nv_bfloat16*>(q_nope),
                    reinterpret_cast<__nv_bfloat16*>(q_pe), status);
}
