// Cache write for new positions ("KV compression" page: the key-value
// down-projection code excerpt, and its Explanation: 576 cached values per
// position).
//
//   cw_gemm_kernel     split-K partial products of kv = x W_KVa on tcgen05:
//                      D^T[o, r] = sum_i W_KVa[i][o] x[r][i] with the 576
//                      output features as M (5 tiles of 128, last one ragged),
//                      the rows as N and K = 7168 cut into 28 chunks of 256.
//   cw_finalize_kernel sum of the chunks, RMSNorm of the 512-wide latent
//                      (fp32), interleaved RoPE of the 64-wide rotary key at
//                      the row's position, bf16 store into the cache.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "host_util.h"

namespace shla {

namespace cw {
constexpr int kDim = 7168, kOut = 576, kLat = 512;
constexpr int KCH = 256;                  // K per CTA
constexpr int NKCH = kDim / KCH;          // 28 chunks
constexpr int MT = 5;                     // output tiles of 128 (576 = 4.5 x 128)
}  // namespace cw

template <typename T>
DEV T* cw_align1024(T* p) {
  return reinterpret_cast<T*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// grid (5 output tiles, 28 K chunks, row blocks of NB); 128 threads.
template <int NB>
__global__ void __launch_bounds__(128) cw_gemm_kernel(const __nv_bfloat16* __restrict__ x,
                                                       const __nv_bfloat16* __restrict__ w,
                                                       int rows, float* __restrict__ part,
                                                       int32_t* status) {
  using namespace cw;
  constexpr uint32_t NCOLS = NB <= 32 ? 32 : NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = cw_align1024(smem_raw);
  const uint32_t sA = smem_u32(smem);       // [2 o-atoms][256 i][128 B] = 64 KB, MN-major
  const uint32_t sB = sA + 65536;           // [4 i-atoms][NB rows][128 B], K-major
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int mt = blockIdx.x, kc = blockIdx.y, r0 = blockIdx.z * NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();  // the finalize kernel may be scheduled (it waits for this grid)

  if (warp == 0) {
    tmem_alloc(&tmem_base, NCOLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init_cluster();
  }
  // A: W_KVa[kc*256 + i][mt*128 + 8*ch .. +8], zero past the 576 outputs
  for (int q = tid; q < KCH * 16; q += 128) {
    const int i = q >> 4, ch = q & 15;
    const int o = mt * 128 + ch * 8;
    const bool in = o < kOut;
    cp_async_16(sA + (ch >> 3) * 32768 + sw128_off(i, ch & 7),
                w + (size_t)(kc * KCH + i) * kOut + (in ? o : 0), in ? 16u : 0u);
  }
  // B: x[r0 + n][kc*256 + 8*ch .. +8]
  for (int q = tid; q < NB * 32; q += 128) {
    const int n = q >> 5, ch = q & 31, r = r0 + n;
    const bool in = r < rows;
    cp_async_16(sB + (ch >> 3) * (NB * 128) + sw128_off(n, ch & 7),
                x + (size_t)(in ? r : 0) * kDim + kc * KCH + ch * 8, in ? 16u : 0u);
  }
  cp_async_wait_all();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, NB, 1, 0);
#pragma unroll
    for (int ks = 0; ks < KCH / 16; ++ks) {
      const uint64_t ad = smem_desc(sA + ks * 2048, 32768, 1024, kSwizzle128B);
      const uint64_t bd =
          smem_desc(sB + (ks >> 2) * (NB * 128) + (ks & 3) * 32, 16, 1024, kSwizzle128B);
      tc_mma(tmem, ad, bd, idesc, ks > 0);
    }
    tc_commit(&bar);
  }
  __syncwarp();
  const bool ok = warp_wait(&bar, 0, nullptr, status);
  tc_fence_after();
  if (ok) {
    const int o = mt * 128 + warp * 32 + lane;
#pragma unroll 1
    for (int n0 = 0; n0 < NB; n0 += 16) {
      uint32_t r[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + n0, r);
      tc_wait_ld();
      if (o < kOut) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int rr = r0 + n0 + j;
          if (rr < rows) part[((size_t)kc * rows + rr) * kOut + o] = __uint_as_float(r[j]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

// one CTA (256 threads) per written row
__global__ void __launch_bounds__(256) cw_finalize_kernel(
    const float* __restrict__ part, int rows, const __nv_bfloat16* __restrict__ norm_w, float eps,
    const float* __restrict__ rope, int S, int start_pos, __nv_bfloat16* c_kv, long long ckv_bs,
    int ckv_rs, __nv_bfloat16* k_pe, long long kpe_bs, int kpe_rs) {
  using namespace cw;
  __shared__ float kv[kOut];
  __shared__ float red[8];
  const int r = blockIdx.x;
  const int b = r / S, s = r - b * S;
  const int pos = start_pos + s;
  const int tid = threadIdx.x;
  pdl_wait();  // the GEMM's partials (a no-op when launched without programmatic dependence)
  float ss = 0.f;
  for (int f = tid; f < kOut; f += 256) {
    // the chunks in order; all their loads in flight together
    float v[NKCH];
#pragma unroll
    for (int c = 0; c < NKCH; ++c) v[c] = part[((size_t)c * rows + r) * kOut + f];
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < NKCH; ++c) acc += v[c];
    kv[f] = acc;
    if (f < kLat) ss += acc * acc;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((tid & 31) == 0) red[tid >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += red[i];
  const float inv = 1.0f / sqrtf(tot / kLat + eps);
  __nv_bfloat16* crow = c_kv + (size_t)b * ckv_bs + (size_t)pos * ckv_rs;
  for (int f = tid; f < kLat; f += 256)
    crow[f] = __float2bfloat16_rn(kv[f] * inv * __bfloat162float(norm_w[f]));
  if (tid < 32) {
    const float a = kv[kLat + 2 * tid], bb = kv[kLat + 2 * tid + 1];
    const float cs = rope[(s * 32 + tid) * 2], sn = rope[(s * 32 + tid) * 2 + 1];
    __nv_bfloat16* prow = k_pe + (size_t)b * kpe_bs + (size_t)pos * kpe_rs;
    prow[2 * tid] = __float2bfloat16_rn(a * cs - bb * sn);
    prow[2 * tid + 1] = __float2bfloat16_rn(a * sn + bb * cs);
  }
}

template <int NB>
static int launch_cw_gemm(const __nv_bfloat16* x, const __nv_bfloat16* w, int rows, float* part,
                          cudaStream_t st) {
  const int smem = 65536 + NB * 512 + 1024;
  static std::atomic<unsigned long long> attr_done{0};
  if (int e = ensure_smem_attr(cw_gemm_kernel<NB>, smem, &attr_done)) return e;
  dim3 grid(cw::MT, cw::NKCH, (rows + NB - 1) / NB);
  cw_gemm_kernel<NB><<<grid, 128, smem, st>>>(x, w, rows, part, nullptr);
  return launch_status();
}

}  // namespace shla

using namespace shla;

extern "C" size_t mla_cache_write_workspace_bytes(int rows) {
  if (rows < 1) return 0;
  return round_up((size_t)cw::NKCH * rows * cw::kOut * sizeof(float), 256);
}

extern "C" int mla_cache_write(const mla_bf16_t* x, const mla_bf16_t* w_kva,
                               const mla_bf16_t* norm_w, float eps, const float* rope, int B,
                               int S, int start_pos, mla_bf16_t* c_kv, int64_t ckv_bstride,
                               int ckv_rstride, mla_bf16_t* k_pe, int64_t kpe_bstride,
                               int kpe_rstride, int T, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !w_kva || !norm_w || !rope || !c_kv || !k_pe) return MLA_ERR_NULL;
  if (B < 1 || S < 1 || (long long)B * S > 4096 || T < 1 || start_pos < 0 ||
      (long long)start_pos + S > T || ckv_rstride < 512 || kpe_rstride < 64 || ckv_bstride < 0 ||
      kpe_bstride < 0 || !(eps >= 0.f))
    return MLA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w_kva) || !aligned16(rope) || !aligned16(c_kv) ||
      !aligned16(k_pe))
    return MLA_ERR_ALIGN;
  const int rows = B * S;
  if (!ws || !aligned256(ws) || ws_bytes < mla_cache_write_workspace_bytes(rows))
    return MLA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  cudaStream_t st = as_stream(stream);
  float* part = static_cast<float*>(ws);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(w_kva);
  int e;
  if (rows <= 16) e = launch_cw_gemm<16>(xb, wb, rows, part, st);
  else if (rows <= 32) e = launch_cw_gemm<32>(xb, wb, rows, part, st);
  else if (rows <= 64) e = launch_cw_gemm<64>(xb, wb, rows, part, st);
  else if (rows <= 128) e = launch_cw_gemm<128>(xb, wb, rows, part, st);
  else e = launch_cw_gemm<256>(xb, wb, rows, part, st);
  if (e) return e;
  // programmatic serialisation: the finalize kernel is scheduled while the
  // GEMM drains and waits for it before reading the partials
  return launch_pdl(cw_finalize_kernel, dim3(rows), dim3(256), 0, st, (const float*)part, rows,
                    reinterpret_cast<const __nv_bfloat16*>(norm_w), eps, rope, S, start_pos,
                    reinterpret_cast<__nv_bfloat16*>(c_kv), (long long)ckv_bstride, ckv_rstride,
                    reinterpret_cast<__nv_bfloat16*>(k_pe), (long long)kpe_bstride, kpe_rstride);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the cache write.
//
// For callers that cannot allocate device memory at the point of the call:
// code running inside CUDA graph node callbacks or other library callbacks,
// runtimes that forbid allocation in their decode loop, and embedders whose
// memory is owned by another allocator they cannot call into.  The split-K
// partial products then go to a fixed, file-scope device array instead of a
// caller workspace.
//
// The array holds partials for at most MLA_NOALLOC_MAX_ROWS rows
// (28 x 64 x 576 floats = 4,128,768 bytes) on every GPU that loads this
// library, until the process exits.  Its host-side name is only a stand-in:
// the device address is looked up with cudaGetSymbolAddress once per device,
// by the first call made with that device current, and looked up again when
// the device's context is no longer the one the address was taken in (after
// cudaDeviceReset, the old address points at freed memory).
// ---------------------------------------------------------------------------
namespace shla {
namespace noalloc {
constexpr int kMaxRows = MLA_NOALLOC_MAX_ROWS;
static __device__ __align__(256) float g_scratch[cw::NKCH * kMaxRows * cw::kOut];

static std::mutex g_mu;
static float* g_addr[64] = {nullptr};
static unsigned long long g_ctx_id[64] = {0};  // context the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// unique id of the calling thread's current context (0 when there is none);
// driver ids are never reused within a process
static unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = []() -> CtxGetCurrentFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(f);
    cudaGetLastError();
    return nullptr;
  }();
  static const CtxGetIdFn get_id = []() -> CtxGetIdFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetIdFn>(f);
    cudaGetLastError();
    return nullptr;
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// device address of g_scratch for the current device (set-up on first use)
static int scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long id = current_context_id();
  if (!g_addr[dev] || id == 0 || id != g_ctx_id[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    g_addr[dev] = static_cast<float*>(p);
    // the symbol lookup made the device's context current if none was
    g_ctx_id[dev] = current_context_id();
  }
  *out = g_addr[dev];
  return MLA_OK;
}
}  // namespace noalloc
}  // namespace shla

extern "C" int mla_cache_write_noalloc(const mla_bf16_t* x, const mla_bf16_t* w_kva,
                                       const mla_bf16_t* norm_w, float eps, const float* rope,
                                       int B, int S, int start_pos, mla_bf16_t* c_kv,
                                       int64_t ckv_bstride, int ckv_rstride, mla_bf16_t* k_pe,
                                       int64_t kpe_bstride, int kpe_rstride, int T,
                                       void* stream) {
  if (!x || !w_kva || !norm_w || !rope || !c_kv || !k_pe) return MLA_ERR_NULL;
  if (B < 1 || S < 1 || (long long)B * S > noalloc::kMaxRows || T < 1 || start_pos < 0 ||
      (long long)start_pos + S > T || ckv_rstride < 512 || kpe_rstride < 64 || ckv_bstride < 0 ||
      kpe_bstride < 0 || !(eps >= 0.f))
    return MLA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w_kva) || !aligned16(rope) || !aligned16(c_kv) ||
      !aligned16(k_pe))
    return MLA_ERR_ALIGN;
  if (int e = check_device()) return e;
  float* part = nullptr;
  if (int e = noalloc::scratch_for_current_device(&part)) return e;
  const int rows = B * S;
  cudaStream_t st = as_stream(stream);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(w_kva);
  // every element of the partial buffer that the finalize step reads is
  // written by the GEMM step of the same call, so nothing needs clearing
  int e;
  if (rows <= 16) e = launch_cw_gemm<16>(xb, wb, rows, part, st);
  else if (rows <= 32) e = launch_cw_gemm<32>(xb, wb, rows, part, st);
  else e = launch_cw_gemm<64>(xb, wb, rows, part, st);
  if (e) return e;
  cw_finalize_kernel<<<rows, 256, 0, st>>>(
      part, rows, reinterpret_cast<const __nv_bfloat16*>(norm_w), eps, rope, S, start_pos,
      reinterpret_cast<__nv_bfloat16*>(c_kv), ckv_bstride, ckv_rstride,
      reinterpret_cast<__nv_bfloat16*>(k_pe), kpe_bstride, kpe_rstride);
  return launch_status();
}
