// Weight-streaming projections of the attention block, and the output
// projection ("Mix and project" page: the output projection wo, the only step
// that mixes heads; its parameter table gives 16,384 x 7,168 = 117,440,512
// weights):
//
//   Delta[b, n] = sum_k x[b, k] W_O[n, k],   x = O[b] flattened head-major
//
// with O [B, 128, 128] bf16 (the decode output), W_O [7168, 16384] bf16 stored
// [out, in], Delta [B, 7168] bf16.  These projections read a large weight for
// a few MB of activations, so they are HBM-bound on the weight.
//
//   xwt_kernel       swap-AB GEMM on tcgen05: D^T[n, b] with 128 rows of W as
//                    M, the batch as N (up to 128 per block), K in chunks of 128
//                    (two 64-wide swizzle atoms, so each W row is read 256
//                    contiguous bytes at a time) through a 3-stage TMA ring.  Persistent CTAs take equal
//                    slices of the flattened (row tile, K chunk) list, so every
//                    SM streams the same number of weight bytes; a slice covers
//                    the end of one row tile and the start of the next, each
//                    part ("segment") ending with an fp32 partial in its slot
//                    of the workspace (see xwt.h).
//   xwt_finish_bf16  sums the slots of each row tile in slot order (a fixed
//                    order: the result does not depend on timing) and rounds
//                    to bf16.
#include <cuda_runtime.h>

#include "common.cuh"
#include "host_util.h"
#include "xwt.h"

namespace shla {
namespace xwt {

constexpr int KA = 64;              // K per 128-byte swizzle atom of bf16 (one TMA box)
constexpr int AT = 2;               // atoms per stage: 256 contiguous bytes of each W row
constexpr int KC = KA * AT;         // K per chunk (one ring stage)
constexpr int NST = 3;              // ring depth: 96 KB of weight in flight per SM
constexpr int ATOM = 16384;         // 128 rows x 128 bytes
constexpr int STAGE = 2 * AT * ATOM;  // W atoms (128 W rows x KC), then X atoms (128 batch rows)
constexpr int SMEM_BYTES = NST * STAGE + 1024;
constexpr int NTHREADS = 192;       // warps 0-3 epilogue, warp 4 loads, warp 5 MMA + TMEM

// TMA tiled load of one box into this CTA's shared memory at (x, y), bytes counted on bar
DEV void tma_load_tile(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

struct Bars {
  uint64_t full[NST], empty[NST];
  uint64_t seg_done[2];   // segment k's products in accumulator k & 1 have completed
  uint64_t tmem_free[2];  // the epilogue has read accumulator k & 1 (128 threads)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

}  // namespace xwt

// ---------------------------------------------------------------------------
// D^T[n, b] = sum_k W[n, k] X[b, k] over this CTA's slice of (row tile,
// K chunk) units, for batch rows [b0, b0 + 128).
//   A = W rows (M = 128, K = 64 per chunk), K-major, 128-byte swizzle
//   B = X rows (N = 128 batch rows),         K-major, 128-byte swizzle
// Rows of the B box beyond B hold stale data; only their own columns of D
// are affected, and those are not stored.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(xwt::NTHREADS, 1)
    xwt_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
               float* __restrict__ part, int B, int a_rows, XwtSched sch, int32_t* status) {
  using namespace xwt;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));  // swizzle atoms: 1 KB aligned
  const uint32_t sbase = smem_u32(smem);
  __shared__ Bars bars;
  volatile int* abort = &bars.abort;
  const int c = blockIdx.x, b0 = blockIdx.y * 128;
  const int u0 = sch.bnd(c), u1 = sch.bnd(c + 1);
  const int nch = sch.nch;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 5) {
    tmem_alloc(&bars.tmem_base, 256);  // two 128-column accumulators
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars.full[s], 1);   // the loader's expect_tx arrival + bytes
      mbar_init(&bars.empty[s], 1);  // MMA commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.seg_done[i], 1);
      mbar_init(&bars.tmem_free[i], 128);
    }
    mbar_init(&bars.drain, 1);
    bars.abort = 0;
    fence_mbarrier_init_cluster();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 4) {
    // ---------------- loads ----------------
    if (lane == 0) {
      int issued = 0;
      int m = u0 / nch, ch = u0 - m * nch, s = 0, ph = 0;  // tile, chunk, stage, its phase
      // The weight is not written by the kernel before this one on the
      // stream: the first stages' weight boxes load before waiting for it.
      const int npre = min(NST, u1 - u0);
      for (int i = 0, mm = m, cc = ch; i < npre; ++i) {
        mbar_arrive_expect_tx(&bars.full[i], AT * (ATOM + 128 * a_rows));
#pragma unroll
        for (int a = 0; a < AT; ++a)
          tma_load_tile(sbase + i * STAGE + a * ATOM, &map_w, cc * KC + a * KA, mm * 128,
                        &bars.full[i]);
        if (++cc == nch) {
          cc = 0;
          ++mm;
        }
      }
      pdl_wait();  // X may be the previous kernel's output
#pragma unroll 1
      for (int u = u0; u < u1; ++u) {
        const uint32_t st = sbase + s * STAGE;
        if (u - u0 >= npre) {
          if (!mbar_wait(&bars.empty[s], ph ^ 1, abort, status)) break;
          mbar_arrive_expect_tx(&bars.full[s], AT * (ATOM + 128 * a_rows));
#pragma unroll
          for (int a = 0; a < AT; ++a)
            tma_load_tile(st + a * ATOM, &map_w, ch * KC + a * KA, m * 128, &bars.full[s]);
        }
#pragma unroll
        for (int a = 0; a < AT; ++a)
          tma_load_tile(st + (AT + a) * ATOM, &map_x, ch * KC + a * KA, b0, &bars.full[s]);
        issued = u - u0 + 1;
        if (++ch == nch) {
          ch = 0;
          ++m;
        }
        if (++s == NST) {
          s = 0;
          ph ^= 1;
        }
      }
      // on an abort, loads still in flight land before the CTA can leave
      for (int i = max(0, issued - NST); i < issued; ++i)
        mbar_wait(&bars.full[i % NST], (i / NST) & 1, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t hi = desc_hi(1024, kSwizzle128B);
      int seg = 0, ch = u0 % nch, s = 0, ph = 0;  // segment, chunk, stage, its phase
#pragma unroll 1
      for (int u = u0; u < u1; ++u) {
        const bool first = u == u0 || ch == 0, last = u == u1 - 1 || ch == nch - 1;
        const int acc = seg & 1;
        if (!mbar_wait(&bars.full[s], ph, abort, status)) break;
        // segment seg reuses accumulator seg & 1 once the epilogue has read
        // segment seg - 2 from it
        if (first && seg >= 2 && !mbar_wait(&bars.tmem_free[acc], ((seg >> 1) - 1) & 1, abort, status))
          break;
        tc_fence_after();
        const uint32_t la = desc_lo(sbase + s * STAGE, 16);
        const uint32_t lb = desc_lo(sbase + s * STAGE + AT * ATOM, 16);
        const uint32_t d = tmem + acc * 128;
        if (first)
          tc_mma_c<false>(d, desc_join(la, hi), desc_join(lb, hi), idesc);
        else
          tc_mma_c<true>(d, desc_join(la, hi), desc_join(lb, hi), idesc);
#pragma unroll
        for (int ks = 1; ks < KC / 16; ++ks) {  // atom ks / 4 (1024 in units of 16 B), K16 step ks % 4
          const uint32_t off = (ks >> 2) * (ATOM >> 4) + (ks & 3) * 2;
          tc_mma_c<true>(d, desc_join(la + off, hi), desc_join(lb + off, hi), idesc);
        }
        tc_commit(&bars.empty[s]);
        if (last) {
          tc_commit(&bars.seg_done[acc]);
          ++seg;
        }
        if (++ch == nch) ch = 0;
        if (++s == NST) {
          s = 0;
          ph ^= 1;
        }
      }
      pdl_trigger();  // all products issued: the finishing kernel may be scheduled
      // everything issued so far has finished before TMEM is released
      tc_commit(&bars.drain);
      mbar_wait(&bars.drain, 0, nullptr, status);
    }
    __syncwarp();
  } else if (u1 > u0) {
    // ---------------- epilogue (warps 0-3: TMEM lane = row of the tile) ----------------
    // segment k of the slice is row tile m0 + k; its partial goes to slot
    // c - c_first(m), 32 consecutive rows per store
    const int m0 = u0 / nch, m1 = (u1 - 1) / nch;
    const int nl = warp * 32 + lane;
#pragma unroll 1
    for (int m = m0, seg = 0; m <= m1; ++m, ++seg) {
      const int acc = seg & 1;
      if (!warp_wait(&bars.seg_done[acc], (seg >> 1) & 1, abort, status)) break;
      tc_fence_after();
      const int slot = c - sch.c_first(m);
      float* dst = part + (size_t)(m * sch.slots + slot) * B * 128 + nl;
#pragma unroll 1
      for (int col = 0; col < 128; col += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + acc * 128 + col, r);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int b = b0 + col + j;
          if (b < B) dst[(size_t)b * 128] = __uint_as_float(r[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.tmem_free[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Y[b, n0 .. n0+7] = bf16(sum over the slots of row tile n0 / 128, in slot
// order).  grid (B, ceil(n_out / 1024)), 128 threads of 8 outputs each.
__global__ void __launch_bounds__(128) xwt_finish_bf16(const float* __restrict__ part,
                                                        XwtSched sch, int B, int n_out,
                                                        __nv_bfloat16* __restrict__ out) {
  const int b = blockIdx.x;
  const int n0 = (blockIdx.y * 128 + threadIdx.x) * 8;
  if (n0 >= n_out) return;
  const int m = n0 / 128, nl = n0 % 128;
  const int used = sch.c_last(m) - sch.c_first(m) + 1;
  pdl_wait();  // the partials of the GEMM before this kernel
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  xwt_sum_slots<4>(part, sch, m, nl, b, B, 0, 1, used, acc);
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(out + (size_t)b * n_out + n0) = o;
}

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------
typedef CUresult (*XwtEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static XwtEncodeFn xwt_encode() {
  // looked up once (a function-local static is initialised thread-safely)
  static const XwtEncodeFn fn = []() -> XwtEncodeFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<XwtEncodeFn>(f);
    cudaGetLastError();
    return nullptr;
  }();
  return fn;
}

// 2-D map over a row-major [rows][cols] bf16 matrix, boxes of 64 x box_rows
static int xwt_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  XwtEncodeFn fn = xwt_encode();
  if (!fn) return MLA_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)xwt::KA, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

XwtSched xwt_plan(int n_out, int k_in) {
  XwtSched s;
  s.nch = k_in / xwt::KC;
  s.tot = (n_out / 128) * s.nch;
  s.nc = s.tot < kXwtCtas ? s.tot : kXwtCtas;
  s.slots = 1;
  for (int m = 0; m < n_out / 128; ++m) {
    const int used = s.c_last(m) - s.c_first(m) + 1;
    if (used > s.slots) s.slots = used;
  }
  return s;
}

size_t xwt_part_bytes(const XwtSched& plan, int n_out, int B) {
  return (size_t)(n_out / 128) * plan.slots * B * 128 * sizeof(float);
}

int xwt_gemm(const void* w, int n_out, int k_in, const void* x, int B, float* part,
             const XwtSched& plan, int32_t* status, cudaStream_t st, bool pdl) {
  const int rows = B < 128 ? B : 128;
  alignas(64) CUtensorMap map_w, map_x;
  if (int e = xwt_map(&map_w, w, n_out, k_in, 128)) return e;
  if (int e = xwt_map(&map_x, x, B, k_in, rows)) return e;
  static std::atomic<unsigned long long> attr_done{0};
  if (int e = ensure_smem_attr(xwt_kernel, xwt::SMEM_BYTES, &attr_done)) return e;
  const dim3 grid(plan.nc, (B + 127) / 128);
  if (pdl)
    return launch_pdl(xwt_kernel, grid, dim3(xwt::NTHREADS), xwt::SMEM_BYTES, st, map_w, map_x,
                      part, B, rows, plan, status);
  xwt_kernel<<<grid, xwt::NTHREADS, xwt::SMEM_BYTES, st>>>(map_w, map_x, part, B, rows, plan,
                                                            status);
  return launch_status();
}

namespace oproj {
constexpr int K_IN = 128 * 128;  // 16384 inputs: 128 heads x 128 value dims, head-major
constexpr int N_OUT = 7168;      // model dimension
}  // namespace oproj

}  // namespace shla

using namespace shla;

extern "C" int mla_xwt_plan(int n_out, int k_in, int32_t* plan, int32_t* first_last) {
  if (!plan) return MLA_ERR_NULL;
  if (n_out < 128 || k_in < xwt::KC || n_out % 128 || k_in % xwt::KC) return MLA_ERR_SHAPE;
  const XwtSched s = xwt_plan(n_out, k_in);
  plan[0] = s.tot;
  plan[1] = s.nc;
  plan[2] = s.nch;
  plan[3] = s.slots;
  if (first_last) {
    for (int m = 0; m < n_out / 128; ++m) {
      first_last[2 * m] = s.c_first(m);
      first_last[2 * m + 1] = s.c_last(m);
    }
  }
  return MLA_OK;
}

extern "C" size_t mla_out_proj_workspace_bytes(int B) {
  if (B < 1 || B > 65535) return 0;
  const XwtSched plan = xwt_plan(oproj::N_OUT, oproj::K_IN);
  return round_up(xwt_part_bytes(plan, oproj::N_OUT, B), 256);
}

extern "C" int mla_out_proj(const mla_bf16_t* O, const mla_bf16_t* w_o, int B, mla_bf16_t* delta,
                            void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  if (!O || !w_o || !delta) return MLA_ERR_NULL;
  if (B < 1 || B > 65535) return MLA_ERR_SHAPE;
  if (!aligned16(O) || !aligned16(w_o) || !aligned16(delta)) return MLA_ERR_ALIGN;
  if (!ws || !aligned256(ws) || ws_bytes < mla_out_proj_workspace_bytes(B))
    return MLA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  const XwtSched plan = xwt_plan(oproj::N_OUT, oproj::K_IN);
  cudaStream_t st = as_stream(stream);
  float* part = static_cast<float*>(ws);
  if (int e = xwt_gemm(w_o, oproj::N_OUT, oproj::K_IN, O, B, part, plan, status, st, false))
    return e;
  return launch_pdl(xwt_finish_bf16, dim3(B, (oproj::N_OUT + 1023) / 1024), dim3(128), 0, st,
                    part, plan, B, oproj::N_OUT, reinterpret_cast<__nv_bfloat16*>(delta));
}
