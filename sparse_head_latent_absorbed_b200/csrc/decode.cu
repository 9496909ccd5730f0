// Absorbed sparse MLA decode for sm_100a ("Mix and project" page, decode
// branch, model.py 590-606).  Three kernels on the caller's stream:
//
//   fold_kernel      q~ = q_nope W_UK per head (tcgen05, latent as M, batch as N)
//   core_kernel      per (batch row, key split), a 2-CTA cluster: gather the
//                    selected cache rows, S = Q~ K^T with the 128 heads as M,
//                    fp32 online softmax, O~ += P V.  CTA r of the pair owns
//                    latent columns [256r, 256r+256) and rotary columns
//                    [32r, 32r+32); the two partial score tiles are summed
//                    through distributed shared memory.
//   merge_uv_kernel  log-sum-exp merge of the splits, then O = O~ W_UV^T per
//                    head (tcgen05, value dim as M, batch as N)
#include <math.h>

#include "common.cuh"
#include "host_util.h"

namespace shla {

constexpr int kH = 128, kC = 512, kR = 64, kDn = 128, kDv = 128;

template <typename T>
DEV T* align1024(T* p) {
  return reinterpret_cast<T*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ===========================================================================
// K1: fold W_UK into the queries.  D^T[c, b] = sum_d W_UK[h][d][c] q_nope[b][h][d]
//   A = W_UK[h] tile (M = 128 latent columns, K = d), MN-major (c contiguous)
//   B = q_nope rows  (N = batch rows,        K = d), K-major
// grid (4 latent tiles, 128 heads, batch blocks of NB); 128 threads.
// ===========================================================================
template <int NB>
__global__ void __launch_bounds__(128) fold_kernel(const __nv_bfloat16* __restrict__ q_nope,
                                                    const __nv_bfloat16* __restrict__ wkv_b,
                                                    __nv_bfloat16* __restrict__ q_tilde, int B,
                                                    int32_t* status) {
  constexpr uint32_t NCOLS = NB <= 32 ? 32 : NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sA = smem_u32(smem);          // [2 atoms][128 d][128 B]  = 32 KB
  const uint32_t sB = sA + 32768;              // [2 katoms][NB rows][128 B]
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int ct = blockIdx.x, h = blockIdx.y, b0 = blockIdx.z * NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    tmem_alloc(&tmem_base, NCOLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init_cluster();
  }
  for (int q = tid; q < 128 * 16; q += 128) {
    const int d = q >> 4, ch = q & 15;
    cp_async_16(sA + (ch >> 3) * 16384 + sw128_off(d, ch & 7),
                wkv_b + ((size_t)h * 256 + d) * kC + ct * 128 + ch * 8, 16);
  }
  for (int q = tid; q < NB * 16; q += 128) {
    const int n = q >> 4, ch = q & 15, b = b0 + n;
    const bool in = b < B;
    cp_async_16(sB + (ch >> 3) * (NB * 128) + sw128_off(n, ch & 7),
                q_nope + ((size_t)(in ? b : 0) * kH + h) * kDn + ch * 8, in ? 16u : 0u);
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
    for (int ks = 0; ks < 8; ++ks) {
      const uint64_t ad = smem_desc(sA + ks * 2048, 16384, 1024, kSwizzle128B);
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
    const int c = ct * 128 + warp * 32 + lane;
#pragma unroll 1
    for (int n0 = 0; n0 < NB; n0 += 16) {
      uint32_t r[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + n0, r);
      tc_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int b = b0 + n0 + j;
        if (b < B)
          q_tilde[((size_t)b * kH + h) * kC + c] = __float2bfloat16_rn(__uint_as_float(r[j]));
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

// ===========================================================================
// K2: sparse attention core on a 2-CTA cluster
//
// Warp roles per CTA (288 threads):
//   warps 0-3  softmax: one thread per head row (TMEM lane); exchange of the
//              partial score tile with the peer CTA through DSMEM, running
//              max / sum, P (bf16) into shared memory, O rescaling
//   warps 4-7  gather: cp.async of this CTA's 288 columns of each selected
//              cache row into a NST-deep ring of key tiles
//   warp 8     TMEM owner and MMA issuer (one thread)
// Per key tile j (KT keys):  S_j = Q~_half K_j_half^T (M=128, N=KT, K=288)
// into one of two TMEM score buffers; after the softmax, O_half += P_j V_j_half
// (M=128, N=256, K=KT) where V is the same shared-memory tile read MN-major.
// ===========================================================================
namespace core {
constexpr int KT = 32;                       // keys per tile
constexpr int NST = 6;                       // gather ring depth
constexpr int NTHREADS = 288;
constexpr int OFF_QC = 0;                    // Q~ latent half: 4 atoms x 128 rows x 128 B
constexpr int OFF_QR = 65536;                // q_pe half: 128 rows x 64 B (64 B swizzle)
constexpr int OFF_ST = 73728;                // key tiles
constexpr int ST_ATOM = KT * 128;            // one 64-column latent atom of a tile
constexpr int ST_KR = 4 * ST_ATOM;           // rotary part of a tile (64 B swizzle)
constexpr int ST_BYTES = ST_KR + KT * 64;
constexpr int OFF_P = OFF_ST + NST * ST_BYTES;   // P: 128 rows x KT bf16 (64 B swizzle)
constexpr int P_BYTES = 128 * KT * 2;
constexpr int OFF_XS = OFF_P + P_BYTES;          // two buffers of exchanged partial scores
constexpr int XS_STRIDE = KT * 4 + 16;           // padded fp32 row
constexpr int XS_BYTES = 128 * XS_STRIDE;
constexpr int OFF_END = OFF_XS + 2 * XS_BYTES;
constexpr uint32_t XS_TX_BYTES = 128 * KT * 4;   // partial scores received per tile
constexpr int SMEM_BYTES = OFF_END + 1024;       // + alignment slack
constexpr uint32_t TMEM_COLS = 512;              // S0 @0, S1 @KT, O half @256
constexpr float kRescaleThreshold = 8.0f;        // log2 units
constexpr int PER_PRODUCER = KT * 36 / 128;      // 16-byte chunks per gather thread per tile
static_assert(KT * 36 % 128 == 0, "gather split");
static_assert(ST_BYTES % 1024 == 0 && OFF_ST % 1024 == 0 && OFF_P % 512 == 0, "alignment");
static_assert(SMEM_BYTES + 256 <= 232448, "shared memory budget");

struct Params {
  const __nv_bfloat16* q_tilde;   // [B][128][512]
  const __nv_bfloat16* q_pe;      // [B][128][64]
  const __nv_bfloat16* c_kv;
  long long ckv_bs;
  int ckv_rs;
  const __nv_bfloat16* k_pe;
  long long kpe_bs;
  int kpe_rs;
  int T;
  const int32_t* topk;
  int k;
  const int32_t* end_pos;
  int B, splits, tiles_per_split, ntiles;
  float scale_log2;               // softmax scale * log2(e)
  __nv_bfloat16* opart;           // [B][splits][128][512], normalised per split
  float* lse;                     // [B][splits][128], log2 units of scaled scores
  int32_t* status;
};

struct Bars {
  uint64_t full[NST], empty[NST], s_full[2], s_empty[2], p_full, o_done, xs_full[2], xs_free[2],
      drain;
  uint32_t tmem_base;
  int abort;
};

DEV bool key_valid(int v, int lim) { return v >= 0 && v < lim; }

}  // namespace core

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(core::NTHREADS, 1)
    core_kernel(const core::Params p) {
  using namespace core;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  __shared__ Bars bars;
  volatile int* abort = &bars.abort;

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cid = blockIdx.x >> 1;
  const int b = cid / p.splits;
  const int sp = cid - b * p.splits;
  const int tile0 = sp * p.tiles_per_split;
  const int nt = min(p.ntiles, tile0 + p.tiles_per_split) - tile0;
  const int lim = min(p.end_pos[b], p.T);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  const int32_t* topk_b = p.topk + (size_t)b * p.k;

  if (warp == 8) {
    tmem_alloc(&bars.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars.full[s], 128);
      mbar_init(&bars.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_empty[i], 128);
      mbar_init(&bars.xs_full[i], 1);    // own expect_tx arrival + the peer's st.async bytes
      mbar_init(&bars.xs_free[i], 4);    // one arrival per softmax warp of the peer
    }
    mbar_init(&bars.p_full, 128);
    mbar_init(&bars.o_done, 1);
    mbar_init(&bars.drain, 1);
    bars.abort = 0;
    fence_mbarrier_init_cluster();
    // first use of each exchange buffer: expect one tile of partial scores
    mbar_arrive_expect_tx(&bars.xs_full[0], XS_TX_BYTES);
    mbar_arrive_expect_tx(&bars.xs_full[1], XS_TX_BYTES);
  }
  // this CTA's half of Q~ (latent) and of q_pe (rotary)
  for (int q = tid; q < 128 * 36; q += NTHREADS) {
    const int h = q / 36, ch = q - h * 36;
    if (ch < 32)
      cp_async_16(sbase + OFF_QC + (ch >> 3) * 16384 + sw128_off(h, ch & 7),
                  p.q_tilde + ((size_t)b * kH + h) * kC + rank * 256 + ch * 8, 16);
    else
      cp_async_16(sbase + OFF_QR + sw64_off(h, ch - 32),
                  p.q_pe + ((size_t)b * kH + h) * kR + rank * 32 + (ch - 32) * 8, 16);
  }
  cp_async_wait_all();
  fence_proxy_async_smem();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp >= 4 && warp < 8) {
    // ---------------- gather ----------------
    const int pt = tid - 128;
    int bad = 0;
    const __nv_bfloat16* ckv_b = p.c_kv + (size_t)b * p.ckv_bs + rank * 256;
    const __nv_bfloat16* kpe_b = p.k_pe + (size_t)b * p.kpe_bs + rank * 32;
    int key[PER_PRODUCER], ch[PER_PRODUCER], v[PER_PRODUCER];
#pragma unroll
    for (int i = 0; i < PER_PRODUCER; ++i) {
      const int q = pt + 128 * i;
      key[i] = q / 36;
      ch[i] = q - key[i] * 36;
      const int j = tile0 * KT + key[i];
      v[i] = j < p.k ? topk_b[j] : -1;
    }
#pragma unroll 1
    for (int jj = 0; jj < nt; ++jj) {
      const int s = jj % NST;
      if (!mbar_wait(&bars.empty[s], ((jj / NST) & 1) ^ 1, abort, p.status)) break;
      const uint32_t stage = sbase + OFF_ST + s * ST_BYTES;
#pragma unroll
      for (int i = 0; i < PER_PRODUCER; ++i) {
        const bool ok = key_valid(v[i], lim);
        if (rank == 0 && ch[i] == 0 && !ok && v[i] != -1) ++bad;
        const long long vv = ok ? v[i] : 0;
        const void* src;
        uint32_t dst;
        if (ch[i] < 32) {
          src = ckv_b + vv * p.ckv_rs + ch[i] * 8;
          dst = stage + (ch[i] >> 3) * ST_ATOM + sw128_off(key[i], ch[i] & 7);
        } else {
          src = kpe_b + vv * p.kpe_rs + (ch[i] - 32) * 8;
          dst = stage + ST_KR + sw64_off(key[i], ch[i] - 32);
        }
        cp_async_16(dst, src, ok ? 16u : 0u);
      }
      cp_async_arrive_noinc(&bars.full[s]);
      // indices of the next tile, loaded while this one is in flight
      if (jj + 1 < nt) {
#pragma unroll
        for (int i = 0; i < PER_PRODUCER; ++i) {
          const int j = (tile0 + jj + 1) * KT + key[i];
          v[i] = j < p.k ? topk_b[j] : -1;
        }
      }
    }
    cp_async_wait_all();
    if (bad && p.status) atomicAdd(p.status + 1, bad);
  } else if (warp == 8) {
    // ---------------- MMA issuer ----------------
    // Event loop: a score tile is computed as soon as its keys have landed
    // and a score buffer is free (up to two tiles ahead of the softmax); a
    // value product as soon as its P is in shared memory.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, KT, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      const uint32_t qc = sbase + OFF_QC, qr = sbase + OFF_QR, pb = sbase + OFF_P;
      int qk = 0, pv = 0, idle = 0;
      uint64_t t_last = globaltimer_ns();
#pragma unroll 1
      while (pv < nt) {
        bool did = false;
        if (qk < nt && mbar_test(&bars.full[qk % NST], (qk / NST) & 1) &&
            mbar_test(&bars.s_empty[qk & 1], ((qk >> 1) & 1) ^ 1)) {
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t st = sbase + OFF_ST + (qk % NST) * ST_BYTES;
          const uint32_t d = tmem + (qk & 1) * KT;
#pragma unroll
          for (int ks = 0; ks < 16; ++ks) {
            const uint64_t ad =
                smem_desc(qc + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd =
                smem_desc(st + (ks >> 2) * ST_ATOM + (ks & 3) * 32, 16, 1024, kSwizzle128B);
            tc_mma(d, ad, bd, idesc_qk, ks > 0);
          }
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t ad = smem_desc(qr + ks * 32, 16, 512, kSwizzle64B);
            const uint64_t bd = smem_desc(st + ST_KR + ks * 32, 16, 512, kSwizzle64B);
            tc_mma(d, ad, bd, idesc_qk, 1);
          }
          tc_commit(&bars.s_full[qk & 1]);
          ++qk;
          did = true;
        }
        if (pv < qk && mbar_test(&bars.p_full, pv & 1)) {
          tc_fence_after();
          const int s = pv % NST;
          const uint32_t st = sbase + OFF_ST + s * ST_BYTES;
#pragma unroll
          for (int ks = 0; ks < KT / 16; ++ks) {
            const uint64_t ad = smem_desc(pb + ks * 32, 16, 512, kSwizzle64B);
            const uint64_t bd = smem_desc(st + ks * 2048, ST_ATOM, 1024, kSwizzle128B);
            tc_mma(tmem + 256, ad, bd, idesc_pv, (pv > 0 || ks > 0) ? 1u : 0u);
          }
          tc_commit(&bars.o_done);
          tc_commit(&bars.empty[s]);
          ++pv;
          did = true;
        }
        if (did) {
          idle = 0;
        } else if (++idle >= 64) {
          idle = 0;
          const uint64_t now = globaltimer_ns();
          if (*abort) break;
          if (now - t_last > kWaitLimitNs) {
            *abort = 1;
            report_timeout(p.status);
            break;
          }
        }
        if (did) t_last = globaltimer_ns();
      }
      // everything issued so far has finished before TMEM is released
      tc_commit(&bars.drain);
      mbar_wait(&bars.drain, 0, nullptr, p.status);
    }
    __syncwarp();
  } else {
    // ---------------- softmax (one thread per head row) ----------------
    const int h = tid;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // exchange buffer / barrier i sits at +i*XS_BYTES / +i*8 from buffer 0 in
    // both CTAs, so the peer addresses follow from one mapa each
    const uint32_t xs_row0 = sbase + OFF_XS + h * XS_STRIDE;
    const uint32_t xs_peer_row0 = mapa_shared(xs_row0, peer);
    const uint32_t xs_full_peer0 = mapa_shared(smem_u32(&bars.xs_full[0]), peer);
    // (each exchange buffer's xs_full phase expects XS_TX_BYTES from the peer)
    const uint32_t xs_free_peer0 = mapa_shared(smem_u32(&bars.xs_free[0]), peer);
    const uint32_t prow = sbase + OFF_P;
    float m_used = -INFINITY, l = 0.f;
    float sn[KT];  // own partial scores of the tile after the current one
    bool alive = true;

    // own partial of tile t: TMEM -> registers -> peer's exchange buffer
    auto fetch_send = [&](int t) -> bool {
      const int b2 = t & 1;
      if (!warp_wait(&bars.s_full[b2], (t >> 1) & 1, abort, p.status)) return false;
      tc_fence_after();
      {
        uint32_t r[16];
#pragma unroll
        for (int c = 0; c < KT; c += 16) {
          tmem_ld16(tmem + lane_base + b2 * KT + c, r);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) sn[c + i] = __uint_as_float(r[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.s_empty[b2]);
      if (!warp_wait<true>(&bars.xs_free[b2], ((t >> 1) & 1) ^ 1, abort, p.status)) return false;
#pragma unroll
      for (int i = 0; i < KT; i += 4)
        st_async_v4(xs_peer_row0 + b2 * XS_BYTES + i * 4, sn[i], sn[i + 1], sn[i + 2], sn[i + 3],
                    xs_full_peer0 + b2 * 8);
      return true;
    };

    int vpre = (tile0 * KT + lane < p.k) ? topk_b[tile0 * KT + lane] : -1;
    alive = fetch_send(0);
#pragma unroll 1
    for (int jj = 0; jj < nt && alive; ++jj) {
      const uint32_t valid = __ballot_sync(0xffffffffu, key_valid(vpre, lim));
      if (jj + 1 < nt) {
        const int j = (tile0 + jj + 1) * KT + lane;
        vpre = j < p.k ? topk_b[j] : -1;
      }
      float s[KT];
#pragma unroll
      for (int i = 0; i < KT; ++i) s[i] = sn[i];
      if (jj + 1 < nt && !fetch_send(jj + 1)) { alive = false; break; }

      // add the peer's partial scores (other latent half) of this tile
      const int b2 = jj & 1;
      if (!warp_wait<true>(&bars.xs_full[b2], (jj >> 1) & 1, abort, p.status)) { alive = false; break; }
#pragma unroll
      for (int i = 0; i < KT; i += 4) {
        float4 o;
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(o.x), "=f"(o.y), "=f"(o.z), "=f"(o.w)
                     : "r"(xs_row0 + b2 * XS_BYTES + i * 4));
        s[i] += o.x;
        s[i + 1] += o.y;
        s[i + 2] += o.z;
        s[i + 3] += o.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(xs_free_peer0 + b2 * 8);
      // next use of this buffer (tile jj + 2): expect the peer's bytes again
      if (tid == 0 && jj + 2 < nt) mbar_arrive_expect_tx(&bars.xs_full[b2], XS_TX_BYTES);

      // scale, mask, running max (log2 domain)
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < KT; ++i) {
        s[i] = ((valid >> i) & 1u) ? s[i] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[i]);
      }
      const float m_new = fmaxf(m_used, mt);
      const bool rescale = m_new > m_used + kRescaleThreshold;
      if (jj > 0) {
        if (!warp_wait(&bars.o_done, (jj - 1) & 1, abort, p.status)) { alive = false; break; }
        tc_fence_after();
      }
      const float alpha = rescale ? fast_exp2(m_used - m_new) : 1.f;
      l *= alpha;
      if (jj > 0 && __any_sync(0xffffffffu, rescale)) {
        // warp-collective: rows that keep their maximum scale by 1
        uint32_t r[16];
#pragma unroll 1
        for (int c = 0; c < 256; c += 16) {
          const uint32_t ta = tmem + lane_base + 256 + c;
          tmem_ld16(ta, r);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st16(ta, r);
        }
        tc_wait_st();
      }
      if (rescale) m_used = m_new;
      // P = 2^(s - m) in bf16; the row sum adds the rounded values
      const bool live = m_used != -INFINITY;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < KT / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float e0 = live ? fast_exp2(s[c * 8 + 2 * i] - m_used) : 0.f;
          const float e1 = live ? fast_exp2(s[c * 8 + 2 * i + 1] - m_used) : 0.f;
          const __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
          const float2 back = __bfloat1622float2(pr);
          psum += back.x + back.y;
          w[i] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        st_shared_v4(prow + sw64_off(h, c), w[0], w[1], w[2], w[3]);
      }
      l += psum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars.p_full);
    }
    // epilogue: this CTA's latent half of O~ / l, and (rank 0) the row's log-sum-exp
    if (__all_sync(0xffffffffu, alive && !*abort)) {
      if (warp_wait(&bars.o_done, (nt - 1) & 1, abort, p.status)) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16* dst =
            p.opart + (((size_t)b * p.splits + sp) * kH + h) * kC + rank * 256;
        uint32_t r[16];
#pragma unroll 1
        for (int c = 0; c < 256; c += 16) {
          tmem_ld16(tmem + lane_base + 256 + c, r);
          tc_wait_ld();
          uint4 lo, hi;
          lo.x = pack_bf16x2(__uint_as_float(r[0]) * inv, __uint_as_float(r[1]) * inv);
          lo.y = pack_bf16x2(__uint_as_float(r[2]) * inv, __uint_as_float(r[3]) * inv);
          lo.z = pack_bf16x2(__uint_as_float(r[4]) * inv, __uint_as_float(r[5]) * inv);
          lo.w = pack_bf16x2(__uint_as_float(r[6]) * inv, __uint_as_float(r[7]) * inv);
          hi.x = pack_bf16x2(__uint_as_float(r[8]) * inv, __uint_as_float(r[9]) * inv);
          hi.y = pack_bf16x2(__uint_as_float(r[10]) * inv, __uint_as_float(r[11]) * inv);
          hi.z = pack_bf16x2(__uint_as_float(r[12]) * inv, __uint_as_float(r[13]) * inv);
          hi.w = pack_bf16x2(__uint_as_float(r[14]) * inv, __uint_as_float(r[15]) * inv);
          *reinterpret_cast<uint4*>(dst + c) = lo;
          *reinterpret_cast<uint4*>(dst + c + 8) = hi;
        }
        if (rank == 0)
          p.lse[((size_t)b * p.splits + sp) * kH + h] = l > 0.f ? m_used + log2f(l) : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  // neither CTA leaves while its peer may still touch its shared memory
  cluster_sync_all();
}

// ===========================================================================
// K3: merge the key splits and apply W_UV.
//   D^T[d, b] = sum_c W_UV[h][d][c] O~[b][h][c]
//   A = W_UV[h] (M = 128 value dims, K = c), K-major
//   B = merged O~ rows (N = batch rows, K = c), K-major, built in shared memory
// grid (128 heads, batch blocks of NB); 256 threads; K in 4 chunks of 128.
// ===========================================================================
template <int NB>
__global__ void __launch_bounds__(256) merge_uv_kernel(const __nv_bfloat16* __restrict__ wkv_b,
                                                        const __nv_bfloat16* __restrict__ opart,
                                                        const float* __restrict__ lse, int B,
                                                        int splits, __nv_bfloat16* __restrict__ O,
                                                        int32_t* status) {
  constexpr uint32_t NCOLS = NB <= 32 ? 32 : NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sA = smem_u32(smem);               // [2 katoms][128 d][128 B] = 32 KB
  const uint32_t sB = sA + 32768;                   // [2 katoms][NB][128 B]
  float* wts = reinterpret_cast<float*>(smem + 32768 + NB * 256);   // [NB][splits]
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int h = blockIdx.x, b0 = blockIdx.y * NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    tmem_alloc(&tmem_base, NCOLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init_cluster();
  }
  // split weights: w_s = 2^(lse_s - max) / sum
  for (int n = tid; n < NB; n += 256) {
    const int b = b0 + n;
    float* w = wts + n * splits;
    if (b >= B) {
      for (int s = 0; s < splits; ++s) w[s] = 0.f;
      continue;
    }
    float mx = -INFINITY;
    for (int s = 0; s < splits; ++s) mx = fmaxf(mx, lse[((size_t)b * splits + s) * kH + h]);
    float sum = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float e = mx == -INFINITY ? 0.f : exp2f(lse[((size_t)b * splits + s) * kH + h] - mx);
      w[s] = e;
      sum += e;
    }
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int s = 0; s < splits; ++s) w[s] *= inv;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  bool ok = true;
#pragma unroll 1
  for (int kc = 0; kc < 4; ++kc) {
    if (kc > 0) {
      ok = warp_wait(&bar, (kc - 1) & 1, nullptr, status) && ok;
      tc_fence_after();
    }
    for (int q = tid; q < 128 * 16; q += 256) {
      const int d = q >> 4, ch = q & 15;
      cp_async_16(sA + (ch >> 3) * 16384 + sw128_off(d, ch & 7),
                  wkv_b + ((size_t)h * 256 + kDn + d) * kC + kc * 128 + ch * 8, 16);
    }
    // merged O~ chunk: 4 independent 16-byte items per thread in flight
#pragma unroll 1
    for (int q0 = tid; q0 < NB * 16; q0 += 256 * 4) {
      float acc[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
#pragma unroll 1
      for (int s = 0; s < splits; ++s) {
        uint4 v[4];
        float w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = q0 + 256 * u;
          const int n = q >> 4, ch = q & 15, b = b0 + n;
          w[u] = (q < NB * 16 && b < B) ? wts[n * splits + s] : 0.f;
          v[u] = make_uint4(0, 0, 0, 0);
          if (w[u] != 0.f)
            v[u] = ld_global_nc_v4(opart + (((size_t)b * splits + s) * kH + h) * kC + kc * 128 +
                                   ch * 8);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(pv[i]);
            acc[u][2 * i] += w[u] * f.x;
            acc[u][2 * i + 1] += w[u] * f.y;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = q0 + 256 * u;
        if (q < NB * 16) {
          const int n = q >> 4, ch = q & 15;
          st_shared_v4(sB + (ch >> 3) * (NB * 128) + sw128_off(n, ch & 7),
                       pack_bf16x2(acc[u][0], acc[u][1]), pack_bf16x2(acc[u][2], acc[u][3]),
                       pack_bf16x2(acc[u][4], acc[u][5]), pack_bf16x2(acc[u][6], acc[u][7]));
        }
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NB, 0, 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = smem_desc(sA + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        const uint64_t bd =
            smem_desc(sB + (ks >> 2) * (NB * 128) + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        tc_mma(tmem, ad, bd, idesc, (kc > 0 || ks > 0) ? 1u : 0u);
      }
      tc_commit(&bar);
    }
    __syncwarp();
  }
  ok = warp_wait(&bar, 1, nullptr, status) && ok;
  tc_fence_after();
  if (ok) {
    // warps w and w+4 share TMEM lanes 32(w%4).. and split the columns
    const int d = (warp & 3) * 32 + lane;
    const int half = warp >> 2;
    constexpr int PER = NB / 2 < 16 ? 16 : NB / 2;
#pragma unroll 1
    for (int n0 = half * PER; n0 < NB && n0 < (half + 1) * PER; n0 += 16) {
      uint32_t r[16];
      tmem_ld16(tmem + ((uint32_t)((warp & 3) * 32) << 16) + n0, r);
      tc_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int b = b0 + n0 + j;
        if (b < B) O[((size_t)b * kH + h) * kDv + d] = __float2bfloat16_rn(__uint_as_float(r[j]));
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

// ===========================================================================
// host side
// ===========================================================================

constexpr int kMaxSplits = 32;

static int ntiles_of(int k) { return (k + core::KT - 1) / core::KT; }

// Pick how many key splits each batch row gets: balance waves of 2-SM
// clusters against the traffic of the per-split partial outputs.
static int choose_splits(int B, int k, int sm_count) {
  const int ntiles = ntiles_of(k);
  const int pairs = sm_count / 2 > 0 ? sm_count / 2 : 1;
  int best_s = 1;
  double best = 1e300;
  const int smax = ntiles < kMaxSplits ? ntiles : kMaxSplits;
  for (int s = 1; s <= smax; ++s) {
    const int tps = (ntiles + s - 1) / s;
    const int se = (ntiles + tps - 1) / tps;
    const long long clusters = (long long)B * se;
    const long long waves = (clusters + pairs - 1) / pairs;
    const double cost = (double)waves * (tps + 1.0) + 3.5 * se * (double)B / pairs;
    if (cost < best - 1e-9) {
      best = cost;
      best_s = se;
    }
  }
  return best_s;
}

static int sm_count_or_default() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
    return n;
  cudaGetLastError();
  return 148;
}

struct WsLayout {
  size_t q_tilde, opart, lse, total;
};

static WsLayout ws_layout(int B, int splits) {
  WsLayout w;
  w.q_tilde = 0;
  w.opart = round_up(w.q_tilde + (size_t)B * kH * kC * 2, 256);
  w.lse = round_up(w.opart + (size_t)B * splits * kH * kC * 2, 256);
  w.total = round_up(w.lse + (size_t)B * splits * kH * 4, 256);
  return w;
}

template <int NB>
static int launch_fold_nb(const __nv_bfloat16* q_nope, const __nv_bfloat16* wkv_b,
                          __nv_bfloat16* q_tilde, int B, int32_t* status, cudaStream_t st) {
  const int smem = 32768 + NB * 256 + 1024;
  static unsigned long long attr_done = 0;
  if (int e = ensure_smem_attr(fold_kernel<NB>, smem, &attr_done)) return e;
  dim3 grid(4, kH, (B + NB - 1) / NB);
  fold_kernel<NB><<<grid, 128, smem, st>>>(q_nope, wkv_b, q_tilde, B, status);
  return launch_status();
}

static int launch_fold(const __nv_bfloat16* q_nope, const __nv_bfloat16* wkv_b,
                       __nv_bfloat16* q_tilde, int B, int32_t* status, cudaStream_t st) {
  if (B <= 16) return launch_fold_nb<16>(q_nope, wkv_b, q_tilde, B, status, st);
  if (B <= 32) return launch_fold_nb<32>(q_nope, wkv_b, q_tilde, B, status, st);
  if (B <= 64) return launch_fold_nb<64>(q_nope, wkv_b, q_tilde, B, status, st);
  if (B <= 128) return launch_fold_nb<128>(q_nope, wkv_b, q_tilde, B, status, st);
  return launch_fold_nb<256>(q_nope, wkv_b, q_tilde, B, status, st);
}

template <int NB>
static int launch_merge_nb(const __nv_bfloat16* wkv_b, const __nv_bfloat16* opart,
                           const float* lse, int B, int splits, __nv_bfloat16* O,
                           int32_t* status, cudaStream_t st) {
  const int smem = 32768 + NB * 256 + NB * kMaxSplits * 4 + 1024;
  static unsigned long long attr_done = 0;
  if (int e = ensure_smem_attr(merge_uv_kernel<NB>, smem, &attr_done)) return e;
  dim3 grid(kH, (B + NB - 1) / NB);
  merge_uv_kernel<NB><<<grid, 256, smem, st>>>(wkv_b, opart, lse, B, splits, O, status);
  return launch_status();
}

static int launch_merge(const __nv_bfloat16* wkv_b, const __nv_bfloat16* opart, const float* lse,
                        int B, int splits, __nv_bfloat16* O, int32_t* status, cudaStream_t st) {
  if (B <= 16) return launch_merge_nb<16>(wkv_b, opart, lse, B, splits, O, status, st);
  if (B <= 32) return launch_merge_nb<32>(wkv_b, opart, lse, B, splits, O, status, st);
  if (B <= 64) return launch_merge_nb<64>(wkv_b, opart, lse, B, splits, O, status, st);
  if (B <= 128) return launch_merge_nb<128>(wkv_b, opart, lse, B, splits, O, status, st);
  return launch_merge_nb<256>(wkv_b, opart, lse, B, splits, O, status, st);
}

static int check_cache_args(const void* c_kv, int64_t ckv_bstride, int ckv_rstride,
                            const void* k_pe, int64_t kpe_bstride, int kpe_rstride, int T) {
  if (!c_kv || !k_pe) return MLA_ERR_NULL;
  if (T < 1 || ckv_rstride < kC || kpe_rstride < kR || ckv_bstride < 0 || kpe_bstride < 0)
    return MLA_ERR_SHAPE;
  if (!aligned16(c_kv) || !aligned16(k_pe) || (ckv_rstride % 8) || (kpe_rstride % 8) ||
      (ckv_bstride % 8) || (kpe_bstride % 8))
    return MLA_ERR_ALIGN;
  return MLA_OK;
}

}  // namespace shla

using namespace shla;

extern "C" int mla_decode_num_splits(int B, int k) {
  if (B < 1 || k < 1) return 0;
  return choose_splits(B, k, sm_count_or_default());
}

extern "C" size_t mla_decode_workspace_bytes(int B, int k) {
  if (B < 1 || k < 1) return 0;
  return ws_layout(B, choose_splits(B, k, sm_count_or_default())).total;
}

extern "C" int mla_fold_wuk(const mla_bf16_t* q_nope, const mla_bf16_t* wkv_b, int B,
                            mla_bf16_t* q_tilde, void* stream) {
  if (!q_nope || !wkv_b || !q_tilde) return MLA_ERR_NULL;
  if (B < 1 || B > 65535) return MLA_ERR_SHAPE;
  if (!aligned16(q_nope) || !aligned16(wkv_b) || !aligned16(q_tilde)) return MLA_ERR_ALIGN;
  if (int e = check_device()) return e;
  return launch_fold(reinterpret_cast<const __nv_bfloat16*>(q_nope),
                     reinterpret_cast<const __nv_bfloat16*>(wkv_b),
                     reinterpret_cast<__nv_bfloat16*>(q_tilde), B, nullptr, as_stream(stream));
}

static int decode_impl(int phase, const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                       const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv, int64_t ckv_bstride,
                       int ckv_rstride, const mla_bf16_t* k_pe, int64_t kpe_bstride,
                       int kpe_rstride, int T, const int32_t* topk, int k,
                       const int32_t* end_pos, int B, float scale, mla_bf16_t* O, void* ws,
                       size_t ws_bytes, int32_t* status, void* stream) {
  if (phase < 0 || phase > 3) return MLA_ERR_SHAPE;
  if (!q_nope || !q_pe || !wkv_b || !topk || !end_pos || !O) return MLA_ERR_NULL;
  if (int e = check_cache_args(c_kv, ckv_bstride, ckv_rstride, k_pe, kpe_bstride, kpe_rstride, T))
    return e;
  if (B < 1 || B > 65535 || k < 1 || k > 65536) return MLA_ERR_SHAPE;
  if (!aligned16(q_nope) || !aligned16(q_pe) || !aligned16(wkv_b) || !aligned16(O))
    return MLA_ERR_ALIGN;
  if (!ws || !aligned256(ws)) return MLA_ERR_WORKSPACE;
  int sms = 0;
  if (int e = check_device(&sms)) return e;
  const int splits = choose_splits(B, k, sms);
  const WsLayout L = ws_layout(B, splits);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  __nv_bfloat16* q_tilde = reinterpret_cast<__nv_bfloat16*>(wsb + L.q_tilde);
  __nv_bfloat16* opart = reinterpret_cast<__nv_bfloat16*>(wsb + L.opart);
  float* lse = reinterpret_cast<float*>(wsb + L.lse);

  if (phase == 0 || phase == 1) {
    if (int e = launch_fold(reinterpret_cast<const __nv_bfloat16*>(q_nope),
                            reinterpret_cast<const __nv_bfloat16*>(wkv_b), q_tilde, B, status, st))
      return e;
  }

  core::Params p;
  p.q_tilde = q_tilde;
  p.q_pe = reinterpret_cast<const __nv_bfloat16*>(q_pe);
  p.c_kv = reinterpret_cast<const __nv_bfloat16*>(c_kv);
  p.ckv_bs = ckv_bstride;
  p.ckv_rs = ckv_rstride;
  p.k_pe = reinterpret_cast<const __nv_bfloat16*>(k_pe);
  p.kpe_bs = kpe_bstride;
  p.kpe_rs = kpe_rstride;
  p.T = T;
  p.topk = topk;
  p.k = k;
  p.end_pos = end_pos;
  p.B = B;
  p.ntiles = ntiles_of(k);
  p.tiles_per_split = (p.ntiles + splits - 1) / splits;
  p.splits = splits;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.opart = opart;
  p.lse = lse;
  p.status = status;
  if (phase == 0 || phase == 2) {
    static unsigned long long core_attr = 0;
    if (int e = ensure_smem_attr(core_kernel, core::SMEM_BYTES, &core_attr)) return e;
    core_kernel<<<dim3(2 * B * splits), core::NTHREADS, core::SMEM_BYTES, st>>>(p);
    if (int e = launch_status()) return e;
  }
  if (phase == 0 || phase == 3)
    return launch_merge(reinterpret_cast<const __nv_bfloat16*>(wkv_b), opart, lse, B, splits,
                        reinterpret_cast<__nv_bfloat16*>(O), status, st);
  return MLA_OK;
}

extern "C" int mla_decode(const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                          const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv, int64_t ckv_bstride,
                          int ckv_rstride, const mla_bf16_t* k_pe, int64_t kpe_bstride,
                          int kpe_rstride, int T, const int32_t* topk, int k,
                          const int32_t* end_pos, int B, float scale, mla_bf16_t* O, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream) {
  return decode_impl(0, q_nope, q_pe, wkv_b, c_kv, ckv_bstride, ckv_rstride, k_pe, kpe_bstride,
                     kpe_rstride, T, topk, k, end_pos, B, scale, O, ws, ws_bytes, status, stream);
}

extern "C" int mla_decode_phase(int phase, const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                                const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv,
                                int64_t ckv_bstride, int ckv_rstride, const mla_bf16_t* k_pe,
                                int64_t kpe_bstride, int kpe_rstride, int T, const int32_t* topk,
                                int k, const int32_t* end_pos, int B, float scale, mla_bf16_t* O,
                                void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  return decode_impl(phase, q_nope, q_pe, wkv_b, c_kv, ckv_bstride, ckv_rstride, k_pe,
                     kpe_bstride, kpe_rstride, T, topk, k, end_pos, B, scale, O, ws, ws_bytes,
                     status, stream);
}
