// Elementwise and gather entry points of libshla: rotary embedding, the
// decode index mask and the cache-row gather (the last two are test hooks
// that expose steps of the decode path).
#include "common.cuh"
#include "host_util.h"

namespace shla {

// ---------------------------------------------------------------------------
// mla_rope ("Rotated shared key" page, apply_rotary_emb)
// ---------------------------------------------------------------------------

// One thread per (row, pair): rows = B*S*Hx, pairs = 32.
__global__ void rope_kernel(const __nv_bfloat16* __restrict__ x, const float2* __restrict__ rope,
                            int S, int Hx, long long n_pairs, int interleaved,
                            __nv_bfloat16* __restrict__ y) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_pairs;
       i += (long long)gridDim.x * blockDim.x) {
    const int j = static_cast<int>(i & 31);
    const long long row = i >> 5;
    const int s = static_cast<int>((row / Hx) % S);
    const float2 cs = rope[s * 32 + j];
    const __nv_bfloat16* xr = x + row * 64;
    __nv_bfloat16* yr = y + row * 64;
    const int i0 = interleaved ? 2 * j : j;
    const int i1 = interleaved ? 2 * j + 1 : j + 32;
    const float a = __bfloat162float(xr[i0]);
    const float b = __bfloat162float(xr[i1]);
    // (a + i b)(cos + i sin)
    const float re = a * cs.x - b * cs.y;
    const float im = a * cs.y + b * cs.x;
    yr[i0] = __float2bfloat16_rn(re);
    yr[i1] = __float2bfloat16_rn(im);
  }
}

// ---------------------------------------------------------------------------
// index mask / gather (decode-branch selection semantics)
// ---------------------------------------------------------------------------

__device__ __forceinline__ bool index_valid(int v, int lim) { return v >= 0 && v < lim; }

__global__ void index_mask_kernel(const int32_t* __restrict__ topk, int B, int k,
                                  const int32_t* __restrict__ end_pos, int T,
                                  uint8_t* __restrict__ mask, int32_t* status) {
  const long long n = (long long)B * k;
  int bad = 0;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int b = static_cast<int>(i / k);
    const int v = topk[i];
    const int lim = min(end_pos[b], T);
    if (index_valid(v, lim)) {
      mask[(long long)b * T + v] = 1;  // duplicates write the same value
    } else if (v != -1) {
      ++bad;
    }
  }
  if (status && bad) atomicAdd(status + 1, bad);
}

// one warp per selected row: 72 chunks of 16 bytes (64 latent + 8 rotary)
__global__ void gather_rows_kernel(const __nv_bfloat16* __restrict__ c_kv, long long ckv_bs,
                                   int ckv_rs, const __nv_bfloat16* __restrict__ k_pe,
                                   long long kpe_bs, int kpe_rs, int T,
                                   const int32_t* __restrict__ topk, int B, int k,
                                   const int32_t* __restrict__ end_pos,
                                   __nv_bfloat16* __restrict__ rows, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const long long warp = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  int bad = 0;
  for (long long i = warp; i < (long long)B * k; i += nwarps) {
    const int b = static_cast<int>(i / k);
    const int v = topk[i];
    const int lim = min(end_pos[b], T);
    const bool ok = index_valid(v, lim);
    if (!ok && v != -1 && lane == 0) ++bad;
    uint4* dst = reinterpret_cast<uint4*>(rows + i * 576);
    for (int c = lane; c < 72; c += 32) {
      uint4 val = make_uint4(0, 0, 0, 0);
      if (ok) {
        const __nv_bfloat16* src =
            c < 64 ? c_kv + b * ckv_bs + (long long)v * ckv_rs + c * 8
                   : k_pe + b * kpe_bs + (long long)v * kpe_rs + (c - 64) * 8;
        val = ld_global_nc_v4(src);
      }
      dst[c] = val;
    }
  }
  if (status && bad) atomicAdd(status + 1, bad);
}

}  // namespace shla

using namespace shla;

extern "C" const char* mla_status_string(int code) {
  switch (code) {
    case MLA_OK: return "ok";
    case MLA_ERR_NULL: return "a required pointer is NULL";
    case MLA_ERR_SHAPE: return "a size or stride is out of range";
    case MLA_ERR_ALIGN: return "a pointer or stride is not 16-byte aligned";
    case MLA_ERR_WORKSPACE: return "workspace is NULL, misaligned or too small";
    case MLA_ERR_UNSUPPORTED: return "device is not compute capability 10.0 (sm_100a)";
    case MLA_ERR_CUDA: return "a CUDA call or kernel launch failed";
    default: return "unknown status code";
  }
}

extern "C" int mla_rope(const mla_bf16_t* x, const float* rope, int B, int S, int Hx,
                        int interleaved, mla_bf16_t* y, void* stream) {
  if (!x || !rope || !y) return MLA_ERR_NULL;
  if (B < 1 || S < 1 || Hx < 1) return MLA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(y) || !aligned16(rope)) return MLA_ERR_ALIGN;
  if (int e = check_device()) return e;
  const long long n = (long long)B * S * Hx * 32;
  const int threads = 256;
  const long long want = (n + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148LL * 64 ? want : 148LL * 64);
  rope_kernel<<<blocks, threads, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(x), reinterpret_cast<const float2*>(rope), S, Hx,
      n, interleaved, reinterpret_cast<__nv_bfloat16*>(y));
  return launch_status();
}

// ---------------------------------------------------------------------------
// the bounded wait's expiry path
// ---------------------------------------------------------------------------

// Two warps wait, through the waits every kernel of the library uses, on an
// mbarrier that nothing arrives on: each gives up after the limit, flags the
// CTA's abort word and the status word, and the kernel returns.  The second
// warp may also leave through the abort word the first one set.
__global__ void __launch_bounds__(64) wait_limit_kernel(int32_t* status, int32_t* gave_up) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_mbarrier_init_cluster();
  }
  __syncthreads();
  const bool ok = warp_wait(&bar, 0, &abort_word, status);
  if (!ok && (threadIdx.x & 31) == 0) atomicAdd(gave_up, 1);
}

extern "C" int mla_wait_limit_check(int32_t* status, int32_t* gave_up, void* stream) {
  if (!status || !gave_up) return MLA_ERR_NULL;
  if (int e = check_device()) return e;
  wait_limit_kernel<<<1, 64, 0, as_stream(stream)>>>(status, gave_up);
  return launch_status();
}

extern "C" int mla_index_mask(const int32_t* topk, int B, int k, const int32_t* end_pos, int T,
                              uint8_t* mask, int32_t* status, void* stream) {
  if (!topk || !end_pos || !mask) return MLA_ERR_NULL;
  if (B < 1 || k < 1 || T < 1) return MLA_ERR_SHAPE;
  if (int e = check_device()) return e;
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(mask, 0, (size_t)B * T, s) != cudaSuccess) return MLA_ERR_CUDA;
  const long long n = (long long)B * k;
  const int threads = 256;
  const long long want = (n + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148LL * 16 ? want : 148LL * 16);
  index_mask_kernel<<<blocks, threads, 0, s>>>(topk, B, k, end_pos, T, mask, status);
  return launch_status();
}

extern "C" int mla_gather_rows(const mla_bf16_t* c_kv, int64_t ckv_bstride, int ckv_rstride,
                               const mla_bf16_t* k_pe, int64_t kpe_bstride, int kpe_rstride,
                               int T, const int32_t* topk, int B, int k,
                               const int32_t* end_pos, mla_bf16_t* rows, int32_t* status,
                               void* stream) {
  if (!c_kv || !k_pe || !topk || !end_pos || !rows) return MLA_ERR_NULL;
  if (B < 1 || k < 1 || T < 1 || ckv_rstride < 512 || kpe_rstride < 64 || ckv_bstride < 0 ||
      kpe_bstride < 0)
    return MLA_ERR_SHAPE;
  if (!aligned16(c_kv) || !aligned16(k_pe) || !aligned16(rows) || (ckv_rstride % 8) ||
      (kpe_rstride % 8) || (ckv_bstride % 8) || (kpe_bstride % 8))
    return MLA_ERR_ALIGN;
  if (int e = check_device()) return e;
  const long long warps = (long long)B * k;
  const int threads = 256;
  const long long want = (warps * 32 + threads - 1) / threads;
  const int blocks = static_cast<int>(want < 148LL * 32 ? want : 148LL * 32);
  gather_rows_kernel<<<blocks, threads, 0, as_stream(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(c_kv), ckv_bstride, ckv_rstride,
      reinterpret_cast<const __nv_bfloat16*>(k_pe), kpe_bstride, kpe_rstride, T, topk, B, k,
      end_pos, reinterpret_cast<__nv_bfloat16*>(rows), status);
  return launch_status();
}
