// Absorbed sparse MLA decode for sm_100a ("Mix and project" page, the decode
// ("MQA decode") code excerpt).  Up to four kernels on the caller's stream
// (mla_decode_mq first runs two small ones that schedule ragged lists,
// row_tiles_kernel and tile_scan_kernel):
//
//   fold_kernel      q~ = q_nope W_UK per head (tcgen05, latent as M, batch as N)
//   core_kernel      persistent 2-CTA clusters over equal ranges of the
//                    (batch row, key tile) list: TMA gather of the selected
//                    cache rows, S = Q~ K^T with the 128 heads as M, fp32
//                    online softmax, O~ += P V.  CTA r of the pair holds latent
//                    columns [256r, 256r+256) and rotary columns [32r, 32r+32);
//                    the two exchange their fp32 partial scores through
//                    distributed shared memory and both run the same softmax
//                    over all heads.
//   combine_kernel   log-sum-exp merge of the rows split across clusters
//                    (launched only when some row is split)
//   uv_kernel        O = O~ W_UV^T per head on the merged O~ (tcgen05, value
//                    dim as M, batch as N)
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
// One CTA per (latent half, head, batch block of NB rows); 128 threads.  Both
// operands arrive by TMA with the 128 B swizzle in one go: the CTA's half of
// W_UK[h] (two M-tiles of 128 latent columns, 64 KB, each with its own
// barrier so that the first products start while the second tile lands) and
// its batch block of q_nope (two 64-wide atoms of d).  The epilogue of M-tile
// 0 overlaps the products of M-tile 1.
// ===========================================================================
template <int NB>
__global__ void __launch_bounds__(128) fold_kernel(const __grid_constant__ CUtensorMap map_w,
                                                    const __grid_constant__ CUtensorMap map_q,
                                                    __nv_bfloat16* __restrict__ q_tilde, int B,
                                                    int32_t* status) {
  constexpr uint32_t NCOLS = 2 * NB < 32 ? 32 : 2 * NB;  // two accumulators of NB columns
  constexpr uint32_t W_TILE = 2 * 16384;                 // one M-tile: 2 atoms x 128 d x 128 B
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t sA = smem_u32(smem);    // [2 M-tiles][2 atoms][128 d][128 B]
  const uint32_t sB = sA + 2 * W_TILE;   // [2 atoms][NB rows][128 B]
  __shared__ uint64_t bar_q, bar_w[2], bar_mma[2];
  __shared__ uint32_t tmem_base;
  const int half = blockIdx.x, h = blockIdx.y, b0 = blockIdx.z * NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_trigger();  // the attend kernel may start its set-up and first gathers

  if (warp == 0) {
    tmem_alloc(&tmem_base, NCOLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_w[i], 1);
      mbar_init(&bar_mma[i], 1);
    }
    fence_mbarrier_init_cluster();
    mbar_arrive_expect_tx(&bar_q, 2 * NB * 128);
    for (int a = 0; a < 2; ++a)
      tma_load_3d(sB + a * (NB * 128), &map_q, a * 64, h, b0, &bar_q);
    for (int mt = 0; mt < 2; ++mt) {
      mbar_arrive_expect_tx(&bar_w[mt], W_TILE);
      for (int a = 0; a < 2; ++a)
        tma_load_2d(sA + mt * W_TILE + a * 16384, &map_w, half * 256 + mt * 128 + a * 64, h * 256,
                    &bar_w[mt]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  bool ok = true;
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, NB, 1, 0);
    ok = mbar_wait(&bar_q, 0, nullptr, status);
    for (int mt = 0; mt < 2 && ok; ++mt) {
      ok = mbar_wait(&bar_w[mt], 0, nullptr, status);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = smem_desc(sA + mt * W_TILE + ks * 2048, 16384, 1024, kSwizzle128B);
        const uint64_t bd =
            smem_desc(sB + (ks >> 2) * (NB * 128) + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        tc_mma(tmem + mt * NB, ad, bd, idesc, ks > 0);
      }
      tc_commit(&bar_mma[mt]);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;  // (only warp 0's lane 0 issued)
  // epilogue per M-tile: D^T[c][b] through shared memory (the M-tile's own
  // operand area, free once its products are done) as [b][128 c] bf16 rows,
  // then 16-byte stores of q~[b][h][256 half + 128 mt ..]
#pragma unroll 1
  for (int mt = 0; mt < 2; ++mt) {
    const bool done = warp_wait(&bar_mma[mt], 0, nullptr, status);
    tc_fence_after();
    const uint32_t stage = sA + mt * W_TILE;
    if (done) {
      const int cl = warp * 32 + lane;  // this thread's c within the tile
#pragma unroll 1
      for (int n0 = 0; n0 < NB; n0 += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + mt * NB + n0, r);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[j]));
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(stage + (n0 + j) * 256 + cl * 2),
                       "h"(*reinterpret_cast<const unsigned short*>(&v))
                       : "memory");
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (done) {
      for (int q = tid; q < NB * 16; q += 128) {
        const int nn = q >> 4, ch = q & 15, b = b0 + nn;
        if (b >= B) continue;
        const uint4 v = ld_shared_v4(stage + nn * 256 + ch * 16);
        *reinterpret_cast<uint4*>(q_tilde + ((size_t)b * kH + h) * kC + half * 256 + mt * 128 +
                                  ch * 8) = v;
      }
    }
  }
  (void)ok;
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

// ===========================================================================
// K2: sparse attention core, persistent 2-CTA clusters
//
// The flattened list of key tiles (batch row b, tile j of row b) is cut into
// one contiguous range per cluster, so every cluster gets the same number of
// tiles whatever B and k are.  A range covers one or more "segments" (the
// part of one batch row it holds); a segment that is the whole row ends with
// the row's normalised O~, any other segment with a partial output (O~
// normalised by its own sum, plus its log-sum-exp) that the combine kernel
// merges.
//
// CTA r of the pair holds latent columns [256r, 256r+256) and rotary columns
// [32r, 32r+32) of Q~ and of every selected cache row, for all 128 heads.  Per
// key tile (KT keys):
//   S_r  = Q~_r K_r^T        partial scores, M=128 heads, N=KT, K=288 (tcgen05)
//   each CTA sends its partial scores to the peer in fp32 (st.async) and adds
//   the peer's to its own, a + b in one CTA and b + a in the other, which are
//   the same fp32 numbers: both CTAs then scale to log2 units, set invalid
//   keys to -inf and run the same fp32 online softmax, bit for bit (running
//   maximum m, raised lazily once the tile maximum exceeds it by more than 8;
//   P = 2^(s - m) rounded to bf16; row sum l of the fp32 P), so nothing else
//   crosses between them.  The exchange runs in its own warps, a tile ahead
//   of the softmax: they free the score tile as soon as they have read it, so
//   the next score product overlaps the softmax of this one.
//   O_r += P V_r             M=128, N=256, K=KT, A = P from TMEM
// V is the same shared-memory tile as K, read MN-major.
//
// Warp roles (640 threads):
//   warps 0-7   softmax: warp w takes the 16 rows [32q + 16h, +16) of lane
//               quarter q = w % 4, h = w / 4, and all keys of a tile, four
//               threads per row (the 16x256b TMEM fragment order), reading
//               the tile's full scores from shared memory
//   warps 8-11  exchange, for lane quarter q = w - 8: read the partial
//               scores from TMEM, send them to the peer, add the peer's and
//               store the full scores for the softmax warps; load this CTA's
//               half of Q~ for the quarter's rows at each segment start
//   warps 12-18 gather: TMA tile::gather4 of the selected rows
//   warp 19     TMEM owner and MMA issuer (one thread)
// TMEM (512 columns): latent half of Q~ [0,128) as bf16 pairs, the score
// tile [128,192), two P tiles [192,256) as bf16 pairs, O~ (latent half,
// fp32) [256,512).
// ===========================================================================
DEV uint32_t f2u(float x) { return __float_as_uint(x); }
DEV float u2f(uint32_t x) { return __uint_as_float(x); }

namespace core {
constexpr int KT = 64;                       // keys per tile
constexpr int NST = 4;                       // gather ring depth
constexpr int NSOFT = 8;                     // softmax warps
constexpr int SEND_WARP0 = 8;                // sender warps 8-11
constexpr int GATHER_WARP0 = 12;
constexpr int NGATHER = 7;                   // gather warps 12-18
constexpr int MMA_WARP = 19;
constexpr int NTHREADS = 32 * (MMA_WARP + 1);  // 640
constexpr int ST_ATOM = KT * 128;            // one 64-column latent atom of a tile
constexpr int ST_KR = 4 * ST_ATOM;           // rotary part of a tile (64 B swizzle)
constexpr int ST_BYTES = ST_KR + KT * 64;    // 36864
constexpr int OFF_ST = 0;
constexpr int OFF_QR = OFF_ST + NST * ST_BYTES;  // rotary half of Q: 128 rows x 64 B, 64 B swizzle
constexpr int OFF_XS = OFF_QR + 128 * 64;        // the peer's partial scores of a tile
constexpr int XS_BYTES = NSOFT * 8 * 32 * 16;    // [softmax warp][8 chunks][32 lanes][16 B]
constexpr int OFF_FS = OFF_XS + XS_BYTES;        // full scores of a tile, the same layout
constexpr int OFF_BIAS = OFF_FS + XS_BYTES;      // per stage: 0 / -inf per key
constexpr int OFF_ROWSTART = OFF_BIAS + NST * KT * 4;  // per stage: the tile starts its row
constexpr int OFF_END = OFF_ROWSTART + NST * 4;
constexpr int SMEM_BYTES = OFF_END + 1024;       // + alignment slack
constexpr uint32_t XS_TX = XS_BYTES;             // partial scores received per tile
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_Q = 0, T_S = 128, T_P = 192, T_O = 256;
constexpr float kRescaleThreshold = 8.0f;        // log2 units
// register split (the launch gives 96 per thread): softmax 96, exchange 128,
// gather / MMA 80: 2 x 96 + 128 + 2 x 80 = 5 x 96
constexpr int REGS_SOFT = 96, REGS_SEND = 128, REGS_REST = 80;
static_assert(128 * (2 * REGS_SOFT + REGS_SEND + 2 * REGS_REST) <= NTHREADS * 96, "register split");
static_assert(ST_BYTES % 1024 == 0 && OFF_QR % 1024 == 0 && OFF_XS % 16 == 0, "alignment");
static_assert(SMEM_BYTES + 512 <= 232448, "shared memory budget");
static_assert(T_Q + 128 <= T_S && T_S + KT <= T_P && T_P + KT <= T_O && T_O + 256 <= TMEM_COLS,
              "TMEM plan");

// Schedule: tiles [bnd(c), bnd(c+1)) of the flattened list belong to cluster c.
// Uniform: every row has nt tiles and the ranges are equal.  Ragged: row b
// has tstart[b + 1] - tstart[b] >= 1 tiles (its list up to the last tile that
// holds an entry other than -1), and the range boundaries tb[] balance the
// tiles plus a fixed cost per row (each row a cluster starts loads its
// queries and writes its output), computed on the device.
struct Sched {
  int nt;                  // tiles per row (uniform)
  int tot;                 // tiles in all (uniform)
  int nc;                  // clusters (uniform: never more than tot)
  const int32_t* tstart;   // ragged: first tile of each row, B + 1 entries; null: uniform
  const int32_t* tb;       // ragged: first tile of each cluster's range, nc + 1 entries
  __host__ __device__ long long bnd(int c) const {
    return tb ? (long long)tb[c] : (long long)c * tot / nc;
  }
  __host__ __device__ long long row_start(int b) const {
    return tstart ? (long long)tstart[b] : (long long)b * nt;
  }
  __device__ int row_tiles(int b) const { return tstart ? tstart[b + 1] - tstart[b] : nt; }
  // uniform: first / last cluster whose range meets row b
  __host__ __device__ int c_first(int b) const {
    return (int)(((row_start(b) + 1) * nc + tot - 1) / tot) - 1;
  }
  __host__ __device__ int c_last(int b) const {
    return (int)((row_start(b + 1) * nc + tot - 1) / tot) - 1;
  }
  // Partial-output slot (0 or 1) of cluster c for row b.  A cluster holds at
  // most two segments that are not whole rows: its first (the row began at
  // or before the range's start: slot 0) and its last (the row began inside
  // the range and runs past its end: slot 1).
  __host__ __device__ int slot(int c, int b) const { return row_start(b) > bnd(c) ? 1 : 0; }
};
// fixed cost of a row, in tiles, in the ragged schedule's balance: the
// query load and output flush a row costs its cluster (measured on B200
// prefill: 1 prompt x 4096 tokens and 4 x 1024, top-k 2048 and 512, the
// total time is flat between 4 and 6 and rises on either side)
constexpr int kRowCostTiles = 5;

struct Params {
  const __nv_bfloat16* q_tilde;   // [B][128][512]
  const __nv_bfloat16* q_pe;      // [B][128][64]
  long long rows_per_b;           // row-index distance between batch rows in the cache maps
  int q_per_row;                  // query rows per cache batch row (query row r reads row r / q_per_row)
  int T;
  const int32_t* topk;
  int k;
  const int32_t* end_pos;
  int B;
  Sched sch;
  const int32_t* crow;            // ragged: the row that holds tile bnd(c), per cluster
  float scale_log2;               // softmax scale * log2(e)
  __nv_bfloat16* opart;           // [clusters][2 slots][128][512], normalised per segment
  float* lse;                     // [clusters][2 slots][128], log2 units of scaled scores
  __nv_bfloat16* omerged;         // [B][128][512]: O~ of rows held by a single cluster
  int32_t* status;
};

struct Bars {
  uint64_t full[NST], empty[NST];  // gather ring
  uint64_t s_full, s_empty;        // score tile in TMEM / read by the exchange warps
  uint64_t xs_full, xs_free;       // peer's partial scores landed / this CTA's buffer read by the peer
  uint64_t f_full, f_free;         // full scores of a tile stored / read by the softmax warps
  uint64_t p_full[2];              // P of tile t is in TMEM buffer t & 1
  uint64_t o_done[2];              // the value product of tile t has completed
  uint64_t q_ready;                // the segment's Q~ is in TMEM / shared memory
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

DEV bool key_valid(int v, int lim) { return v >= 0 && v < lim; }

// Position of a tile in the flattened list, advanced one tile at a time
// (no division in the loops): batch row, tile within the row, the row's
// tile count and valid-position limit, and the tile's indices (lane l: keys
// l and 32 + l).
struct TileCur {
  int bb, jt, nr, lim, ilo, ihi;
};
// The same position without the limit and the indices.
struct Pos {
  int bb, jt, nr;
};

}  // namespace core

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(core::NTHREADS, 1)
    core_kernel(const core::Params p, const __grid_constant__ CUtensorMap map_c,
                const __grid_constant__ CUtensorMap map_r) {
  using namespace core;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  __shared__ Bars bars;
  volatile int* abort = &bars.abort;

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cid = blockIdx.x >> 1;
  const int t_begin = (int)p.sch.bnd(cid), t_end = (int)p.sch.bnd(cid + 1);
  const int n = t_end - t_begin;  // tiles of this cluster (ragged rows: possibly none)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the merge / W_UV kernels may be scheduled; they take an SM only once
  // this kernel's CTA has left it (it holds the whole register file)
  pdl_trigger();
  const uint32_t sbase = smem_u32(smem);
  // row / tile-in-row of tile 0
  const int bb0 = p.sch.tstart ? ld_global_nc_s32_early(p.crow + cid) : t_begin / p.sch.nt;
  const int jt0 = t_begin - (int)p.sch.row_start(bb0);
  auto tiles_of = [&](int bb) { return bb < p.B ? p.sch.row_tiles(bb) : 1; };
  auto lim_of = [&](int bb) { return min(ld_global_nc_s32_early(p.end_pos + bb), p.T); };
  // the tile after `c` (indices and limit loaded, not yet consumed)
  auto advance = [&](const TileCur& c) {
    TileCur d;
    d.bb = c.bb;
    d.jt = c.jt + 1;
    d.nr = c.nr;
    d.lim = c.lim;
    if (d.jt == d.nr) {
      d.jt = 0;
      ++d.bb;
      d.nr = tiles_of(d.bb);
      d.lim = d.bb < p.B ? lim_of(d.bb) : 0;
    }
    d.ilo = d.ihi = -1;
    if (d.bb < p.B) {
      const int j = d.jt * KT + lane;
      const int32_t* tk = p.topk + (size_t)d.bb * p.k;
      d.ilo = j < p.k ? ld_global_nc_s32_early(tk + j) : -1;
      d.ihi = j + 32 < p.k ? ld_global_nc_s32_early(tk + j + 32) : -1;
    }
    return d;
  };
  auto first_cur = [&]() {
    TileCur c;
    c.bb = bb0;
    c.jt = jt0 - 1;  // advance() from the tile before
    c.nr = tiles_of(bb0);
    c.lim = lim_of(bb0);
    c.ilo = c.ihi = -1;
    return advance(c);
  };
  auto next_pos = [&](Pos c) {
    if (++c.jt == c.nr) {
      c.jt = 0;
      ++c.bb;
      c.nr = tiles_of(c.bb);
    }
    return c;
  };

  if (warp == MMA_WARP) {
    tmem_alloc(&bars.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars.full[s], NGATHER);  // one expect_tx arrival per gather warp + bytes
      mbar_init(&bars.empty[s], 1);       // MMA commit after the tile's value product
    }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.s_empty, 4);
    mbar_init(&bars.xs_full, 1);     // own expect_tx arrival + the peer's st.async bytes
    mbar_init(&bars.xs_free, 4);     // one arrival per exchange warp of the peer
    mbar_init(&bars.f_full, 4);
    mbar_init(&bars.f_free, NSOFT);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.p_full[i], NSOFT);
      mbar_init(&bars.o_done[i], 1);
    }
    mbar_init(&bars.q_ready, 4);
    mbar_init(&bars.drain, 1);
    bars.abort = 0;
    fence_mbarrier_init_cluster();
    mbar_arrive_expect_tx(&bars.xs_full, XS_TX);
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (n == 0) {
    // an empty range (ragged rows, fewer tiles than clusters): nothing to do
  } else if (warp >= GATHER_WARP0 && warp < MMA_WARP) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_REST));
    // ---------------- gather (TMA tile::gather4) ----------------
    // lane l holds the index of key l and key 32 + l of the tile; lanes
    // 0..ng-1 each issue the five loads of one group of four keys
    const int gw = warp - GATHER_WARP0;
    const int ng = (16 - gw + NGATHER - 1) / NGATHER;  // groups of this warp
    constexpr uint32_t GROUP_TX_BYTES = ST_BYTES / 16;
    int bad = 0, issued = 0;
    int base_bb = -1;      // query row whose cache base is in `base`
    long long base = 0;    // first TMA row of that query row's cache batch row
    TileCur cur = first_cur();
#pragma unroll 1
    for (int i = 0; i < n; ++i) {
      const int s = i % NST;
      const bool oka = key_valid(cur.ilo, cur.lim), okb = key_valid(cur.ihi, cur.lim);
      if (rank == 0 && gw == 0) bad += (!oka && cur.ilo != -1) + (!okb && cur.ihi != -1);
      // TMA rows: valid keys map to their cache row, others to row -1 (zero fill)
      if (cur.bb != base_bb) {
        base_bb = cur.bb;
        base = (long long)(cur.bb / p.q_per_row) * p.rows_per_b;
      }
      const int ra = oka ? (int)(base + cur.ilo) : -1;
      const int rb = okb ? (int)(base + cur.ihi) : -1;
      const bool row_start = cur.jt == 0;
      if (i + 1 < n) cur = advance(cur);
      if (!warp_wait(&bars.empty[s], ((i / NST) & 1) ^ 1, abort, p.status)) break;
      if (gw == 0) {
        // the tile's key biases (0 / -inf), read by the softmax warps
        const uint32_t bias = sbase + OFF_BIAS + s * (KT * 4);
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(bias + lane * 4), "f"(oka ? 0.f : -INFINITY)
                     : "memory");
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(bias + (32 + lane) * 4),
                     "f"(okb ? 0.f : -INFINITY)
                     : "memory");
        if (lane == 0)
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(sbase + OFF_ROWSTART + s * 4),
                       "r"(i == 0 || row_start ? 1u : 0u)
                       : "memory");
        __syncwarp();
      }
      if (lane == 0) mbar_arrive_expect_tx(&bars.full[s], ng * GROUP_TX_BYTES);
      __syncwarp();
      const int g = gw + NGATHER * (lane < ng ? lane : 0);  // this lane's group
      const int k0 = 4 * g;                                 // its first key (0..60)
      const int src = k0 & 31;
      const int y0 = __shfl_sync(0xffffffffu, ra, src);
      const int y0b = __shfl_sync(0xffffffffu, rb, src);
      const int y1 = __shfl_sync(0xffffffffu, ra, src + 1);
      const int y1b = __shfl_sync(0xffffffffu, rb, src + 1);
      const int y2 = __shfl_sync(0xffffffffu, ra, src + 2);
      const int y2b = __shfl_sync(0xffffffffu, rb, src + 2);
      const int y3 = __shfl_sync(0xffffffffu, ra, src + 3);
      const int y3b = __shfl_sync(0xffffffffu, rb, src + 3);
      if (lane < ng) {
        const bool hi = k0 >= 32;
        const int r0 = hi ? y0b : y0, r1 = hi ? y1b : y1, r2 = hi ? y2b : y2, r3 = hi ? y3b : y3;
        const uint32_t stage = sbase + OFF_ST + s * ST_BYTES;
#pragma unroll
        for (int a = 0; a < 4; ++a)
          tma_gather4(stage + a * ST_ATOM + k0 * 128, &map_c, rank * 256 + a * 64, r0, r1, r2, r3,
                      &bars.full[s]);
        tma_gather4(stage + ST_KR + k0 * 64, &map_r, rank * 32, r0, r1, r2, r3, &bars.full[s]);
      }
      issued = i + 1;
    }
    // on an abort, the loads still in flight land before the CTA can leave
    // (the waits are bounded and already complete on the normal path)
    for (int t = max(0, issued - NST); t < issued; ++t)
      warp_wait(&bars.full[t % NST], (t / NST) & 1, nullptr, nullptr);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
    if (lane == 0 && bad && p.status) atomicAdd(p.status + 1, bad);
  } else if (warp == MMA_WARP) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_REST));
    // ---------------- MMA issuer ----------------
    // Event loop.  A value product (A = P of tile t from TMEM buffer t & 1)
    // goes first whenever its P is ready; a score product as soon as its keys
    // have landed, the previous score tile has been read and this segment's
    // Q~ is in place.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, KT, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      // descriptors: a stage's low word plus a constant per K-step
      constexpr uint32_t hi_k128 = desc_hi(1024, kSwizzle128B);  // 128 B swizzle
      constexpr uint32_t hi_k64 = desc_hi(512, kSwizzle64B);     // 64 B swizzle
      const uint32_t lo_qr = desc_lo(sbase + OFF_QR, 16);        // rotary half of Q
      int qk = 0, pv = 0, idle = 0, qseg = -1;
      int qs = 0, qph = 0, ps = 0;  // stage of the next score product (and its phase), value product
      uint64_t t_idle = 0;  // when the current idle stretch was first checked (0: not yet)
#pragma unroll 1
      while (pv < n) {
        bool did = false;
        if (pv < qk && mbar_test(&bars.p_full[pv & 1], (pv >> 1) & 1)) {
          tc_fence_after();
          const int s = ps;
          const uint32_t lo = desc_lo(sbase + OFF_ST + s * ST_BYTES, ST_ATOM);  // V, MN-major
          const uint32_t tp = tmem + T_P + (pv & 1) * (KT / 2);
          // the tile starts a segment: its row's first tile, or the range's
          const bool first = ld_shared_u32(sbase + OFF_ROWSTART + s * 4) != 0;
          if (first)
            tc_mma_tmem_a_c<false>(tmem + T_O, tp, desc_join(lo, hi_k128), idesc_pv);
          else
            tc_mma_tmem_a_c<true>(tmem + T_O, tp, desc_join(lo, hi_k128), idesc_pv);
#pragma unroll
          for (int ks = 1; ks < KT / 16; ++ks)
            tc_mma_tmem_a_c<true>(tmem + T_O, tp + ks * 8, desc_join(lo + ks * (2048 >> 4), hi_k128),
                                  idesc_pv);
          tc_commit(&bars.o_done[pv & 1]);
          tc_commit(&bars.empty[s]);
          ++pv;
          if (++ps == NST) ps = 0;
          did = true;
        }
        if (qk < n && mbar_test(&bars.full[qs], qph) &&
            (qk == 0 || mbar_test(&bars.s_empty, (qk - 1) & 1))) {
          const int seg = ld_shared_u32(sbase + OFF_ROWSTART + qs * 4) ? qseg + 1 : qseg;
          if (seg == qseg || mbar_test(&bars.q_ready, seg & 1)) {
            qseg = seg;
            tc_fence_after();
            const uint32_t st = sbase + OFF_ST + qs * ST_BYTES;
            const uint32_t lo = desc_lo(st, 16), lo_r = desc_lo(st + ST_KR, 16);
            const uint32_t ts = tmem + T_S;
            tc_mma_tmem_a_c<false>(ts, tmem + T_Q, desc_join(lo, hi_k128), idesc_qk);
#pragma unroll
            for (int ks = 1; ks < 16; ++ks)
              tc_mma_tmem_a_c<true>(
                  ts, tmem + T_Q + ks * 8,
                  desc_join(lo + (((ks >> 2) * ST_ATOM + (ks & 3) * 32) >> 4), hi_k128), idesc_qk);
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
              tc_mma_c<true>(ts, desc_join(lo_qr + ks * 2, hi_k64), desc_join(lo_r + ks * 2, hi_k64),
                             idesc_qk);
            tc_commit(&bars.s_full);
            ++qk;
            if (++qs == NST) {
              qs = 0;
              qph ^= 1;
            }
            did = true;
          }
        }
        // the time limit runs from the first check of an idle stretch (the
        // timer is read only while nothing is ready)
        if (did) {
          idle = 0;
          t_idle = 0;
        } else if (__nanosleep(20), ++idle >= 64) {
          // (nothing ready: the sleep leaves the issue slots to the softmax warps)
          idle = 0;
          if (*abort) break;
          const uint64_t now = globaltimer_ns();
          if (t_idle == 0) {
            t_idle = now;
          } else if (now - t_idle > kWaitLimitNs) {
            *abort = 1;
            report_timeout(p.status);
            break;
          }
        }
      }
      // everything issued so far has finished before TMEM is released
      tc_commit(&bars.drain);
      mbar_wait(&bars.drain, 0, nullptr, p.status);
    }
    __syncwarp();
  } else if (warp >= SEND_WARP0) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SEND));
    // ---------------- exchange for lane quarter q ----------------
    // The two 16-lane halves of the quarter, in the 16x256b fragment order of
    // the softmax warps q (half 0) and q + 4 (half 1): register 4k+e of half
    // hf is chunk k of softmax warp q + 4 hf.
    const int q4 = warp - SEND_WARP0;
    const uint32_t xs_peer = mapa_shared(sbase + OFF_XS + lane * 16, peer);
    const uint32_t xs_full_peer = mapa_shared(smem_u32(&bars.xs_full), peer);
    const uint32_t xs_free_peer = mapa_shared(smem_u32(&bars.xs_free), peer);
    const uint32_t own_xs = sbase + OFF_XS + lane * 16;
    const uint32_t own_fs = sbase + OFF_FS + lane * 16;
    // the quarter's 32 rows of this CTA's half of Q~ for batch row bb (32x32b
    // shape, one row per thread): latent values into TMEM as bf16 pairs,
    // rotary values into the swizzled shared tile; then q_ready
    auto load_q = [&](int bb) {
      const int h = q4 * 32 + lane;
      const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
      const __nv_bfloat16* qrow = p.q_tilde + ((size_t)bb * kH + h) * kC + rank * 256;
      // two rounds of 16 loads in flight per thread (the row's load is on
      // the path to its first score product)
#pragma unroll 1
      for (int c = 0; c < 4; c += 2) {
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = ld_global_nc_v4(qrow + c * 64 + i * 8);
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            r[4 * i] = v[8 * hc + i].x;
            r[4 * i + 1] = v[8 * hc + i].y;
            r[4 * i + 2] = v[8 * hc + i].z;
            r[4 * i + 3] = v[8 * hc + i].w;
          }
          tmem_st32(tmem + lane_base + T_Q + (c + hc) * 32, r);
        }
      }
      const __nv_bfloat16* rrow = p.q_pe + ((size_t)bb * kH + h) * kR + rank * 32;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 v = ld_global_nc_v4(rrow + c * 8);
        st_shared_v4(sbase + OFF_QR + sw64_off(h, c), v.x, v.y, v.z, v.w);
      }
      fence_proxy_async_smem();
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.q_ready);
    };
    // this thread's part of the next row's queries into L2, a row ahead of
    // its load (the next row starts inside this cluster's range)
    auto prefetch_q = [&](int i, const Pos& c) {
      if (i + c.nr - c.jt >= n) return;
      const int h = q4 * 32 + lane;
      const __nv_bfloat16* qrow = p.q_tilde + ((size_t)(c.bb + 1) * kH + h) * kC + rank * 256;
#pragma unroll
      for (int j = 0; j < 4; ++j) prefetch_l2(qrow + j * 64);
      prefetch_l2(p.q_pe + ((size_t)(c.bb + 1) * kH + h) * kR + rank * 32);
    };
    pdl_wait();  // q~ is the fold kernel's output (the other roles read only inputs)
    load_q(bb0);
    Pos c = {bb0, jt0, tiles_of(bb0)};
    int nx = 0;  // next tile whose exchange buffer is consumed
#pragma unroll 1
    for (int i = 0; i < n; ++i) {
      if (i == 0 || c.jt == 0) prefetch_q(i, c);
      if (!warp_wait(&bars.s_full, i & 1, abort, p.status)) break;
      tc_fence_after();
      uint32_t r[2][32];
      tmem_ld_16x256b_x8(tmem + ((uint32_t)(q4 * 32) << 16) + T_S, r[0]);
      tmem_ld_16x256b_x8(tmem + ((uint32_t)(q4 * 32 + 16) << 16) + T_S, r[1]);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      // relaxed: the tcgen05 loads have completed (waited for above)
      if (lane == 0) mbar_arrive_relaxed(&bars.s_empty);
      // this CTA's partial scores to the peer (its buffer of tile i - 1 read)
      if (!warp_wait<true>(&bars.xs_free, (i & 1) ^ 1, abort, p.status)) break;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          st_async_u4(xs_peer + (q4 + 4 * hf) * 4096 + k * 512, r[hf][4 * k], r[hf][4 * k + 1],
                      r[hf][4 * k + 2], r[hf][4 * k + 3], xs_full_peer);
      // own + peer, in fp32
      if (!warp_wait<true>(&bars.xs_full, i & 1, abort, p.status)) break;
      nx = i + 1;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 v = ld_shared_v4(own_xs + (q4 + 4 * hf) * 4096 + k * 512);
          r[hf][4 * k] = f2u(u2f(r[hf][4 * k]) + u2f(v.x));
          r[hf][4 * k + 1] = f2u(u2f(r[hf][4 * k + 1]) + u2f(v.y));
          r[hf][4 * k + 2] = f2u(u2f(r[hf][4 * k + 2]) + u2f(v.z));
          r[hf][4 * k + 3] = f2u(u2f(r[hf][4 * k + 3]) + u2f(v.w));
        }
      // the sums are computed (so the buffer's loads have returned) before
      // the relaxed arrive below is issued
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int j = 0; j < 32; ++j) asm volatile("" : "+r"(r[hf][j]));
      __syncwarp();
      if (lane == 0) {
        // next use of the buffer (tile i + 1): expect the peer's bytes again,
        // then let the peer write them.  Relaxed: the reads have completed
        // (their values are consumed above), and a release would also wait
        // for the remote stores just issued.
        if (q4 == 0 && i + 1 < n) mbar_arrive_expect_tx_relaxed(&bars.xs_full, XS_TX);
        mbar_arrive_cluster_relaxed(xs_free_peer);
      }
      // the full scores for the softmax warps (their buffer of tile i - 1 read)
      if (!warp_wait(&bars.f_free, (i & 1) ^ 1, abort, p.status)) break;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          st_shared_v4(own_fs + (q4 + 4 * hf) * 4096 + k * 512, r[hf][4 * k], r[hf][4 * k + 1],
                       r[hf][4 * k + 2], r[hf][4 * k + 3]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.f_full);
      // the score tile just finished was the last product that used this
      // segment's Q~ when the tile ends its batch row: load the next row's,
      // after this tile's full scores are out (the softmax and the segment's
      // flush proceed meanwhile)
      if (c.jt == c.nr - 1 && i + 1 < n) load_q(c.bb + 1);
      c = next_pos(c);
    }
    // on an abort, partial scores the peer may still be sending land before
    // the CTA can leave: the armed, unconsumed phase (bounded wait; none
    // remains on the normal path)
    if (nx < n) warp_wait<true>(&bars.xs_full, nx & 1, nullptr, nullptr);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFT));
    // ---------------- softmax: rows [32q + 16h, +16), all keys ----------------
    // Through the 16x256b TMEM shape thread t holds rows t/4 and t/4 + 8 of
    // its 16 and, of each 8-key block j, keys 8j + 2(t%4) and 8j + 2(t%4) + 1:
    // register 4j+e is (row t/4 + 8 (e/2), key 8j + 2(t%4) + e%2).
    const int q4 = warp & 3, hf = warp >> 2;
    const int c4 = lane & 3;
    const int row0 = q4 * 32 + hf * 16 + (lane >> 2), row1 = row0 + 8;
    const uint32_t frag = (uint32_t)(q4 * 32 + hf * 16) << 16;
    const uint32_t fs_own = sbase + OFF_FS + warp * 4096 + lane * 16;
    bool alive = true;

    // the value product of tile t has completed
    auto wait_pv = [&](int t) -> bool {
      if (!warp_wait(&bars.o_done[t & 1], (t >> 1) & 1, abort, p.status)) return false;
      tc_fence_after();
      return true;
    };
    // this thread's two rows of this CTA's half of O~ times a0 / a1
    auto rescale_o = [&](float a0, float a1) {
#pragma unroll 1
      for (int cc = 0; cc < 256; cc += 32) {
        uint32_t r[16];
        const uint32_t ta = tmem + frag + T_O + cc;
        tmem_ld_16x256b_x4(ta, r);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          r[4 * j] = f2u(u2f(r[4 * j]) * a0);
          r[4 * j + 1] = f2u(u2f(r[4 * j + 1]) * a0);
          r[4 * j + 2] = f2u(u2f(r[4 * j + 2]) * a1);
          r[4 * j + 3] = f2u(u2f(r[4 * j + 3]) * a1);
        }
        tmem_st_16x256b_x4(ta, r);
      }
      tc_wait_st();
    };
    float m0 = -INFINITY, m1 = -INFINITY;  // running maxima of the two rows (log2 units)
    float l0 = 0.f, l1 = 0.f;              // this thread's parts of their row sums
    // epilogue of a segment: this thread's rows of this CTA's half of O~ / l
    // into the row's output (a row held by one cluster) or the segment's slot,
    // and (rank 0) the segment's log-sum-exps
    // `partial`: the segment is not its whole row (it began mid-row at the
    // range's start, or its row runs past the range's end); such a segment
    // goes to slot 0 of this cluster when it is the range's first, else to
    // slot 1 (the rule of Sched::slot)
    auto flush = [&](int i_last, int bb, bool partial, int slot1) -> bool {
      float t0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
      t0 += __shfl_xor_sync(0xffffffffu, t0, 2);
      float t1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
      t1 += __shfl_xor_sync(0xffffffffu, t1, 2);
      if (!wait_pv(i_last)) return false;
      const int slot = 2 * cid + slot1;
      const float inv0 = t0 > 0.f ? 1.f / t0 : 0.f;
      const float inv1 = t1 > 0.f ? 1.f / t1 : 0.f;
      __nv_bfloat16* dst0 =
          (!partial ? p.omerged + ((size_t)bb * kH + row0) * kC
                    : p.opart + ((size_t)slot * kH + row0) * kC) +
          rank * 256 + 2 * c4;
      __nv_bfloat16* dst1 = dst0 + 8 * kC;
      uint32_t r[16];
#pragma unroll 1
      for (int cc = 0; cc < 256; cc += 32) {
        tmem_ld_16x256b_x4(tmem + frag + T_O + cc, r);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          *reinterpret_cast<uint32_t*>(dst0 + cc + 8 * j) =
              pack_bf16x2(u2f(r[4 * j]) * inv0, u2f(r[4 * j + 1]) * inv0);
          *reinterpret_cast<uint32_t*>(dst1 + cc + 8 * j) =
              pack_bf16x2(u2f(r[4 * j + 2]) * inv1, u2f(r[4 * j + 3]) * inv1);
        }
      }
      tc_fence_before();
      if (partial && rank == 0 && c4 == 0) {
        float* lse = p.lse + (size_t)slot * kH;
        lse[row0] = t0 > 0.f ? m0 + log2f(t0) : -INFINITY;
        lse[row1] = t1 > 0.f ? m1 + log2f(t1) : -INFINITY;
      }
      return true;
    };
    float x[32];
    Pos c = {bb0, jt0, tiles_of(bb0)};
    int prev_bb = bb0;
    bool open = false;  // the last tile processed is not its row's last
    int nseg = 0;       // segments written out
#pragma unroll 1
    for (int i = 0; i < n && alive; ++i) {
      const int b = i & 1;
      const bool first = i == 0 || c.jt == 0;
      // a new segment: write out the previous one (which ended its row) and
      // restart the running state
      if (first && i > 0) {
        if (!flush(i - 1, prev_bb, nseg == 0 && jt0 > 0, 0)) { alive = false; break; }
        ++nseg;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
      }
      // key biases of the tile (its stage stays in place until the tile's value product)
      if (!warp_wait(&bars.full[i % NST], (i / NST) & 1, abort, p.status)) { alive = false; break; }
      float2 bias[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                     : "=f"(bias[j].x), "=f"(bias[j].y)
                     : "r"(sbase + OFF_BIAS + (i % NST) * (KT * 4) + (8 * j + 2 * c4) * 4));
      // the tile's full scores (exchange warps)
      if (!warp_wait(&bars.f_full, i & 1, abort, p.status)) { alive = false; break; }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint4 v = ld_shared_v4(fs_own + k * 512);
        x[4 * k] = u2f(v.x);
        x[4 * k + 1] = u2f(v.y);
        x[4 * k + 2] = u2f(v.z);
        x[4 * k + 3] = u2f(v.w);
      }
      __syncwarp();
      // release: the exchange warps overwrite the buffer as soon as this arrives
      if (lane == 0) mbar_arrive(&bars.f_free);
      // scale to log2 units, mask (fp32); row maxima
      float mt0 = -INFINITY, mt1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        x[4 * j] = fmaf(x[4 * j], p.scale_log2, bias[j].x);
        x[4 * j + 1] = fmaf(x[4 * j + 1], p.scale_log2, bias[j].y);
        x[4 * j + 2] = fmaf(x[4 * j + 2], p.scale_log2, bias[j].x);
        x[4 * j + 3] = fmaf(x[4 * j + 3], p.scale_log2, bias[j].y);
        mt0 = fmaxf(mt0, fmaxf(x[4 * j], x[4 * j + 1]));
        mt1 = fmaxf(mt1, fmaxf(x[4 * j + 2], x[4 * j + 3]));
      }
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, o));
        mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, o));
      }
      const bool resc0 = mt0 > m0 + kRescaleThreshold, resc1 = mt1 > m1 + kRescaleThreshold;
      if (!first && __any_sync(0xffffffffu, resc0 || resc1)) {
        // O~ must hold the value product of tile i - 1 before it is scaled
        if (!wait_pv(i - 1)) { alive = false; break; }
        rescale_o(resc0 ? fast_exp2(m0 - mt0) : 1.f, resc1 ? fast_exp2(m1 - mt1) : 1.f);
      }
      if (resc0) {
        l0 *= first ? 0.f : fast_exp2(m0 - mt0);
        m0 = mt0;
      }
      if (resc1) {
        l1 *= first ? 0.f : fast_exp2(m1 - mt1);
        m1 = mt1;
      }
      // P buffer b was last read by the value product of tile i - 2
      if (i >= 2 && !wait_pv(i - 2)) { alive = false; break; }
      // P = 2^(s - m) in fp32, rounded to bf16 pairs into TMEM buffer b (the
      // pair of block j lands in P column 4j + c4 of its row)
      {
        const bool live0 = m0 != -INFINITY, live1 = m1 != -INFINITY;
        uint32_t w[16];
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float e0 = live0 ? fast_exp2(x[4 * j] - m0) : 0.f;
          const float e1 = live0 ? fast_exp2(x[4 * j + 1] - m0) : 0.f;
          const float e2 = live1 ? fast_exp2(x[4 * j + 2] - m1) : 0.f;
          const float e3 = live1 ? fast_exp2(x[4 * j + 3] - m1) : 0.f;
          s0 += e0 + e1;
          s1 += e2 + e3;
          w[2 * j] = pack_bf16x2(e0, e1);
          w[2 * j + 1] = pack_bf16x2(e2, e3);
        }
        l0 += s0;
        l1 += s1;
        tmem_st_16x128b_x8(tmem + frag + T_P + b * (KT / 2), w);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[b]);
      prev_bb = c.bb;
      open = c.jt != c.nr - 1;
      c = next_pos(c);
    }
    if (__all_sync(0xffffffffu, alive) && !*abort)
      flush(n - 1, prev_bb, (nseg == 0 && jt0 > 0) || open, nseg == 0 ? 0 : 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  // neither CTA leaves while its peer may still touch its shared memory
  cluster_sync_all();
}

// ===========================================================================
// K3a: merge the segments of the rows that more than one cluster held
//   O~[b,h,:] = sum_s 2^(lse_s - max) O~_s / sum_s 2^(lse_s - max)
// grid (cluster boundaries 1 .. clusters-1, 8 groups of 16 heads); 256
// threads, 4 x 16 bytes each per segment.  Boundary c merges the row that
// holds tile bnd(c) when the boundary falls inside that row and is the row's
// first one; rows held by one cluster were written final by the attend
// kernel.
// ===========================================================================
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ opart,
                                                       const float* __restrict__ lse,
                                                       const core::Sched sch,
                                                       const int32_t* __restrict__ crow,
                                                       __nv_bfloat16* __restrict__ omerged) {
  const int cb = blockIdx.x + 1;
  pdl_trigger();
  // every block waits for the attend kernel, those with nothing to merge
  // too: the W_UV kernel after this one relies on this grid's completion
  // implying the attend kernel's (it reads the rows written final there)
  pdl_wait();
  const long long t = sch.bnd(cb);
  const int b = sch.tb ? ld_global_nc_s32_early(crow + cb) : (int)(t / sch.nt);
  const long long rs = sch.row_start(b), re = sch.row_start(b + 1);
  // the boundary is inside the row, and the one before it is not: cluster
  // cb - 1 holds the row's first tile
  if (rs == t || sch.bnd(cb - 1) > rs) return;
  const int cf = cb - 1;
  const int h = blockIdx.y * 16 + (threadIdx.x >> 4);
  const int c0 = (threadIdx.x & 15) * 8;  // chunks c0, c0 + 128, c0 + 256, c0 + 384
  // the row's segments, in cluster order: slot 1 of cluster cf (slot 0 when
  // the row starts its range), slot 0 of every later cluster whose range
  // starts inside the row and is not empty
  auto holds = [&](int c) { return c == cf || sch.bnd(c) != sch.bnd(c + 1); };
  auto in_row = [&](int c) { return c < sch.nc && (c == cf || sch.bnd(c) < re); };
  auto next_held = [&](int from) {  // the next cluster from `from` on holding a segment, or -1
    int x = from;
    while (in_row(x) && !holds(x)) ++x;
    return in_row(x) ? x : -1;
  };
  const int s0 = 2 * cf + sch.slot(cf, b);
  auto slot_of = [&](int c) { return (size_t)(c == cf ? s0 : 2 * c); };
  const float* lse_h = lse + h;
  const __nv_bfloat16* src = opart + (size_t)h * kC + c0;
  float acc[4][8];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
  float wsum = 0.f;
  auto add = [&](const uint4 (&v)[4], float w) {
    wsum += w;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v[j]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(pv[e]);
        acc[j][2 * e] += w * f.x;
        acc[j][2 * e + 1] += w * f.y;
      }
    }
  };
  // the row's segments in cluster order; up to four (every split row of the
  // workloads here) two at a time, each pair's loads in flight together
  constexpr int kFast = 4;
  int cl[kFast];
  cl[0] = cf;
  cl[1] = next_held(cf + 1);
  cl[2] = cl[1] >= 0 ? next_held(cl[1] + 1) : -1;
  cl[3] = cl[2] >= 0 ? next_held(cl[2] + 1) : -1;
  const int more = cl[3] >= 0 ? next_held(cl[3] + 1) : -1;
  const int np = cl[1] < 0 ? 1 : cl[2] < 0 ? 2 : cl[3] < 0 ? 3 : 4;
  if (more < 0) {
    float l[kFast];
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < kFast; ++q)
      if (q < np) {
        l[q] = lse_h[slot_of(cl[q]) * kH];
        mx = fmaxf(mx, l[q]);
      }
    // two segments at a time, both segments' loads in flight together
#pragma unroll
    for (int q = 0; q < kFast; q += 2) {
      if (q < np) {
        uint4 va[4], vb[4];
        const size_t sa = slot_of(cl[q]);
        const size_t sb = slot_of(q + 1 < np ? cl[q + 1] : cl[q]);
#pragma unroll
        for (int j = 0; j < 4; ++j) va[j] = ld_global_nc_v4(src + sa * kH * kC + j * 128);
#pragma unroll
        for (int j = 0; j < 4; ++j) vb[j] = ld_global_nc_v4(src + sb * kH * kC + j * 128);
        add(va, mx == -INFINITY ? 0.f : exp2f(l[q] - mx));
        if (q + 1 < np) add(vb, mx == -INFINITY ? 0.f : exp2f(l[q + 1] - mx));
      }
    }
  } else {
    // more segments (very small B x k): in cluster order, one after another
    float mx = -INFINITY;
    for (int c2 = cf; c2 >= 0; c2 = next_held(c2 + 1)) mx = fmaxf(mx, lse_h[slot_of(c2) * kH]);
#pragma unroll 1
    for (int c2 = cf; c2 >= 0; c2 = next_held(c2 + 1)) {
      const size_t sl = slot_of(c2);
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = ld_global_nc_v4(src + sl * kH * kC + j * 128);
      add(v, mx == -INFINITY ? 0.f : exp2f(lse_h[sl * kH] - mx));
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* out = omerged + ((size_t)b * kH + h) * kC + c0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 o;
    o.x = pack_bf16x2(acc[j][0] * inv, acc[j][1] * inv);
    o.y = pack_bf16x2(acc[j][2] * inv, acc[j][3] * inv);
    o.z = pack_bf16x2(acc[j][4] * inv, acc[j][5] * inv);
    o.w = pack_bf16x2(acc[j][6] * inv, acc[j][7] * inv);
    *reinterpret_cast<uint4*>(out + j * 128) = o;
  }
}

// ===========================================================================
// Ragged rows (several query rows per cache row: prefill and multi-query
// decode, whose lists end in -1 padding).  Row r needs the tiles up to and
// including the last one that holds an entry other than -1, and at least
// one, so that a row with nothing listed still gets its zero output; the
// tiles after it hold only padding and are not scheduled.
//   row_tiles_kernel   one warp per row, scanning its list from the end
//   tile_scan_kernel   one block: tstart = exclusive prefix sum of the
//                      counts (B + 1 entries) and, per cluster c, the row
//                      that holds tile bnd(c)
// ===========================================================================
__global__ void __launch_bounds__(256) row_tiles_kernel(const int32_t* __restrict__ topk, int k,
                                                         int B, int32_t* __restrict__ cnt) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= B) return;
  const int32_t* row = topk + (size_t)r * k;
  int t = (k + core::KT - 1) / core::KT;
#pragma unroll 1
  for (; t > 1; --t) {
    const int j0 = (t - 1) * core::KT + lane, j1 = j0 + 32;
    const bool listed = (j0 < k && ld_global_nc_s32_early(row + j0) != -1) ||
                        (j1 < k && ld_global_nc_s32_early(row + j1) != -1);
    if (__any_sync(0xffffffffu, listed)) break;
  }
  if (lane == 0) cnt[r] = t;
}

__global__ void __launch_bounds__(1024) tile_scan_kernel(const int32_t* __restrict__ cnt, int B,
                                                          int nc, int32_t* __restrict__ tstart,
                                                          int32_t* __restrict__ tb,
                                                          int32_t* __restrict__ crow) {
  __shared__ int part[1024];
  const int tid = threadIdx.x;
  const int per = (B + 1023) / 1024;
  const int lo = min(B, tid * per), hi = min(B, lo + per);
  int sum = 0;
  for (int r = lo; r < hi; ++r) sum += cnt[r];
  part[tid] = sum;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int run = part[tid] - sum;
  for (int r = lo; r < hi; ++r) {
    tstart[r] = run;
    run += cnt[r];
  }
  const int tot = part[1023];
  if (tid == 0) tstart[B] = tot;
  __syncthreads();  // tstart written by the block is visible to it
  // Cost units: row r spans core::kRowCostTiles units of its own cost, then one
  // unit per tile, from u(r) = tstart[r] + r * core::kRowCostTiles.  Cluster c
  // takes the units [c * U / nc, (c + 1) * U / nc); a range that starts in a
  // row's own units starts at the row's first tile.
  const long long U = (long long)tot + (long long)B * core::kRowCostTiles;
  for (int c = tid; c <= nc; c += 1024) {
    if (c == nc) {
      tb[c] = tot;
      crow[c] = B;
      continue;
    }
    const long long u = (long long)c * U / nc;
    int a = 0, e = B;  // u(a) <= u < u(e)
    while (e - a > 1) {
      const int m = (a + e) >> 1;
      if ((long long)tstart[m] + (long long)m * core::kRowCostTiles <= u) a = m; else e = m;
    }
    const long long into = u - ((long long)tstart[a] + (long long)a * core::kRowCostTiles);
    tb[c] = tstart[a] + (into > core::kRowCostTiles ? (int)(into - core::kRowCostTiles) : 0);
    crow[c] = a;
  }
}

// ===========================================================================
// K3: O = O~ W_UV^T per head, on the merged O~ of each row.
//   D^T[d, b] = sum_c W_UV[h][d][c] O~[b][h][c]
//   A = W_UV[h] (M = 128 value dims, K = c), K-major
//   B = O~ rows (N = batch rows, K = c), K-major
// grid (128 heads, batch blocks of NB); 128 threads; K in 4 chunks of 128,
// double-buffered (cp.async for chunk k+2 while the MMAs of chunk k run).
// ===========================================================================
template <int NB>
__global__ void __launch_bounds__(128) uv_kernel(const __nv_bfloat16* __restrict__ wkv_b,
                                                  const __nv_bfloat16* __restrict__ omerged,
                                                  int B, __nv_bfloat16* __restrict__ O,
                                                  int32_t* status) {
  constexpr uint32_t NCOLS = NB <= 32 ? 32 : NB;
  constexpr uint32_t BUF = 32768 + NB * 256;        // one chunk: A [2 katoms][128][128 B] + B
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t s0 = smem_u32(smem);
  __shared__ uint64_t bar[2];
  __shared__ uint32_t tmem_base;
  const int h = blockIdx.x, b0 = blockIdx.y * NB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    tmem_alloc(&tmem_base, NCOLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbarrier_init_cluster();
  }
  pdl_wait();  // O~ of the attend or combine kernel
  auto load_chunk = [&](int kc) {
    const uint32_t sA = s0 + (kc & 1) * BUF, sB = sA + 32768;
    for (int q = tid; q < 128 * 16; q += 128) {
      const int d = q >> 4, ch = q & 15;
      cp_async_16(sA + (ch >> 3) * 16384 + sw128_off(d, ch & 7),
                  wkv_b + ((size_t)h * 256 + kDn + d) * kC + kc * 128 + ch * 8, 16);
    }
    for (int q = tid; q < NB * 16; q += 128) {
      const int nn = q >> 4, ch = q & 15, b = b0 + nn;
      const bool in = b < B;
      cp_async_16(sB + (ch >> 3) * (NB * 128) + sw128_off(nn, ch & 7),
                  omerged + ((size_t)(in ? b : 0) * kH + h) * kC + kc * 128 + ch * 8,
                  in ? 16u : 0u);
    }
    cp_async_commit();
  };
  load_chunk(0);
  load_chunk(1);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  bool ok = true;
#pragma unroll 1
  for (int kc = 0; kc < 4; ++kc) {
    if (kc < 3) cp_async_wait<1>(); else cp_async_wait<0>();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NB, 0, 0);
      const uint32_t sA = s0 + (kc & 1) * BUF, sB = sA + 32768;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t ad = smem_desc(sA + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        const uint64_t bd =
            smem_desc(sB + (ks >> 2) * (NB * 128) + (ks & 3) * 32, 16, 1024, kSwizzle128B);
        tc_mma(tmem, ad, bd, idesc, (kc > 0 || ks > 0) ? 1u : 0u);
      }
      tc_commit(&bar[kc & 1]);
    }
    __syncwarp();
    if (kc + 2 < 4) {
      // buffer kc&1 is refilled once the MMAs that read it are done
      ok = warp_wait(&bar[kc & 1], (kc >> 1) & 1, nullptr, status) && ok;
      load_chunk(kc + 2);
    }
  }
  // last two commits: chunk 2 (bar[0], phase 1) and chunk 3 (bar[1], phase 1)
  ok = warp_wait(&bar[0], 1, nullptr, status) && ok;
  ok = warp_wait(&bar[1], 1, nullptr, status) && ok;
  tc_fence_after();
  // epilogue: D^T[d][b] through shared memory as [b][128 d] bf16 rows, then
  // 16-byte stores of O[b][h][:]
  const uint32_t stage = s0;
  if (ok) {
    const int d = warp * 32 + lane;
#pragma unroll 1
    for (int n0 = 0; n0 < NB; n0 += 16) {
      uint32_t r[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + n0, r);
      tc_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const __nv_bfloat16 v = __float2bfloat16_rn(__uint_as_float(r[j]));
        asm volatile("st.shared.b16 [%0], %1;" ::"r"(stage + (n0 + j) * 256 + d * 2),
                     "h"(*reinterpret_cast<const unsigned short*>(&v))
                     : "memory");
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (ok) {
    for (int q = tid; q < NB * 16; q += 128) {
      const int nn = q >> 4, ch = q & 15, b = b0 + nn;
      if (b >= B) continue;
      uint4 v;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                   : "r"(stage + nn * 256 + ch * 16));
      *reinterpret_cast<uint4*>(O + ((size_t)b * kH + h) * kDv + ch * 8) = v;
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOLS);
  }
}

// ===========================================================================
// host side
// ===========================================================================

static int ntiles_of(int k) { return (k + core::KT - 1) / core::KT; }

// Clusters of the attend kernel that fit on the device at once (cached per
// device); every cluster is persistent over its range of tiles.
static int max_clusters() {
  // two host threads that both find the entry empty store the same value
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 74;
  }
  if (dev < 64) {
    const int c = cached[dev].load(std::memory_order_acquire);
    if (c > 0) return c;
  }
  int n = 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * 512);
  cfg.blockDim = dim3(core::NTHREADS);
  cfg.dynamicSmemBytes = core::SMEM_BYTES;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaFuncSetAttribute(core_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           core::SMEM_BYTES) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, core_kernel, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      sms = 148;
    }
    n = sms / 2;
  }
  if (dev < 64) cached[dev].store(n, std::memory_order_release);
  return n;
}

static core::Sched make_sched(int B, int k, int clusters) {
  core::Sched s;
  s.nt = ntiles_of(k);
  s.tot = B * s.nt;
  s.nc = clusters < s.tot ? clusters : s.tot;
  s.tstart = nullptr;
  s.tb = nullptr;
  return s;
}

// partial-output slots per batch row: the most clusters that meet one row
static int slots_of(const core::Sched& s, int B) {
  int m = 1;
  for (int b = 0; b < B; ++b) {
    const int u = s.c_last(b) - s.c_first(b) + 1;
    if (u > m) m = u;
  }
  return m;
}

struct WsLayout {
  size_t q_tilde, opart, lse, omerged, cnt, tstart, tb, crow, total;
};

// Partial outputs are held per cluster (two slots each), so their size
// depends on the cluster count, not on B or on how the rows are split.
static WsLayout ws_layout(int B, int clusters) {
  WsLayout w;
  w.q_tilde = 0;
  w.opart = round_up(w.q_tilde + (size_t)B * kH * kC * 2, 256);
  w.lse = round_up(w.opart + (size_t)clusters * 2 * kH * kC * 2, 256);
  w.omerged = round_up(w.lse + (size_t)clusters * 2 * kH * 4, 256);
  w.cnt = round_up(w.omerged + (size_t)B * kH * kC * 2, 256);
  w.tstart = round_up(w.cnt + (size_t)B * 4, 256);
  w.tb = round_up(w.tstart + (size_t)(B + 1) * 4, 256);
  w.crow = round_up(w.tb + (size_t)(clusters + 1) * 4, 256);
  w.total = round_up(w.crow + (size_t)(clusters + 1) * 4, 256);
  return w;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  // looked up once (a function-local static is initialised thread-safely)
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(f);
    cudaGetLastError();
    return nullptr;
  }();
  return fn;
}

// tensor map over a bf16 array: dims / byte strides from the innermost
// dimension, box of `box` elements, 128 B swizzle
static int make_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                    const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return MLA_ERR_CUDA;
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                        strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

template <int NB>
static int launch_fold_nb(const __nv_bfloat16* q_nope, const __nv_bfloat16* wkv_b,
                          __nv_bfloat16* q_tilde, int B, int32_t* status, cudaStream_t st) {
  alignas(64) CUtensorMap map_w, map_q;
  {
    // wkv_b as [128 heads x 256 rows][512 latent]: a box is 128 d-rows of one
    // head by 64 latent columns
    const cuuint64_t dims[2] = {(cuuint64_t)kC, (cuuint64_t)kH * 256};
    const cuuint64_t strides[1] = {(cuuint64_t)kC * 2};
    const cuuint32_t box[2] = {64, 128};
    if (int e = make_map(&map_w, wkv_b, 2, dims, strides, box)) return e;
  }
  {
    // q_nope as [B][128 heads][128 d]: a box is 64 d of one head for NB rows
    const cuuint64_t dims[3] = {(cuuint64_t)kDn, (cuuint64_t)kH, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)kDn * 2, (cuuint64_t)kH * kDn * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)NB};
    if (int e = make_map(&map_q, q_nope, 3, dims, strides, box)) return e;
  }
  const int smem = 2 * 32768 + NB * 256 + 1024;
  static std::atomic<unsigned long long> attr_done{0};
  if (int e = ensure_smem_attr(fold_kernel<NB>, smem, &attr_done)) return e;
  dim3 grid(2, kH, (B + NB - 1) / NB);
  fold_kernel<NB><<<grid, 128, smem, st>>>(map_w, map_q, q_tilde, B, status);
  return launch_status();
}

static int launch_fold(const __nv_bfloat16* q_nope, const __nv_bfloat16* wkv_b,
                       __nv_bfloat16* q_tilde, int B, int32_t* status, cudaStream_t st) {
  if (B <= 16) return launch_fold_nb<16>(q_nope, wkv_b, q_tilde, B, status, st);
  if (B <= 32) return launch_fold_nb<32>(q_nope, wkv_b, q_tilde, B, status, st);
  if (B <= 64) return launch_fold_nb<64>(q_nope, wkv_b, q_tilde, B, status, st);
  return launch_fold_nb<128>(q_nope, wkv_b, q_tilde, B, status, st);
}

template <int NB>
static int launch_uv_nb(const __nv_bfloat16* wkv_b, const __nv_bfloat16* omerged, int B,
                        __nv_bfloat16* O, int32_t* status, cudaStream_t st, bool pdl) {
  const int smem = 2 * (32768 + NB * 256) + 1024;
  static std::atomic<unsigned long long> attr_done{0};
  if (int e = ensure_smem_attr(uv_kernel<NB>, smem, &attr_done)) return e;
  dim3 grid(kH, (B + NB - 1) / NB);
  if (pdl) return launch_pdl(uv_kernel<NB>, grid, dim3(128), smem, st, wkv_b, omerged, B, O, status);
  uv_kernel<NB><<<grid, 128, smem, st>>>(wkv_b, omerged, B, O, status);
  return launch_status();
}

// pdl: launched right after a kernel of the same call (programmatic serialisation)
static int launch_uv(const __nv_bfloat16* wkv_b, const __nv_bfloat16* omerged, int B,
                     __nv_bfloat16* O, int32_t* status, cudaStream_t st, bool pdl) {
  if (B <= 16) return launch_uv_nb<16>(wkv_b, omerged, B, O, status, st, pdl);
  if (B <= 32) return launch_uv_nb<32>(wkv_b, omerged, B, O, status, st, pdl);
  if (B <= 64) return launch_uv_nb<64>(wkv_b, omerged, B, O, status, st, pdl);
  if (B <= 128) return launch_uv_nb<128>(wkv_b, omerged, B, O, status, st, pdl);
  return launch_uv_nb<256>(wkv_b, omerged, B, O, status, st, pdl);
}

// The number of clusters is capped so that no batch row meets more than
// kMaxSlots of them, which bounds the segments the merge of one row reads
// (only matters for very small B x k).
constexpr int kMaxSlots = 32;

static core::Sched schedule_for(int B, int k) {
  int nc = max_clusters();
  core::Sched s = make_sched(B, k, nc);
  while (slots_of(s, B) > kMaxSlots && s.nc > 1) s = make_sched(B, k, s.nc - 1);
  return s;
}

// Ragged rows: the cluster count of the uniform schedule of the same B and
// k; the ranges come from the tile counts on the device (tile_scan_kernel),
// and with fewer tiles than clusters some of them are empty.
static core::Sched ragged_schedule_for(int B, int k, const int32_t* tstart, const int32_t* tb) {
  core::Sched s = schedule_for(B, k);
  s.tot = 0;  // (the ranges come from tb)
  s.tstart = tstart;
  s.tb = tb;
  return s;
}

// 2-D tensor map over cache rows: dims {cols, rows}, row pitch rstride
// elements, box {box_cols, 1} (one row high, as tile::gather4 requires).
static int make_row_map(CUtensorMap* map, const void* base, int cols, unsigned long long rows,
                        int rstride, int box_cols, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return MLA_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)rstride * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, 1};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

static int check_cache_args(const void* c_kv, int64_t ckv_bstride, int ckv_rstride,
                            const void* k_pe, int64_t kpe_bstride, int kpe_rstride, int T) {
  if (!c_kv || !k_pe) return MLA_ERR_NULL;
  if (T < 1 || ckv_rstride < kC || kpe_rstride < kR || ckv_bstride < 0 || kpe_bstride < 0)
    return MLA_ERR_SHAPE;
  if (!aligned16(c_kv) || !aligned16(k_pe) || (ckv_rstride % 8) || (kpe_rstride % 8) ||
      (ckv_bstride % 8) || (kpe_bstride % 8))
    return MLA_ERR_ALIGN;
  // the gather addresses rows as b * (bstride / rstride) + t in both caches
  if (ckv_bstride % ckv_rstride || kpe_bstride % kpe_rstride ||
      ckv_bstride / ckv_rstride != kpe_bstride / kpe_rstride ||
      (ckv_bstride != 0 && ckv_bstride / ckv_rstride < T))
    return MLA_ERR_SHAPE;
  return MLA_OK;
}

}  // namespace shla

using namespace shla;

extern "C" int mla_decode_num_splits(int B, int k) {
  if (B < 1 || k < 1) return 0;
  return slots_of(schedule_for(B, k), B);
}

extern "C" size_t mla_decode_workspace_bytes(int B, int k) {
  if (B < 1 || k < 1) return 0;
  return ws_layout(B, max_clusters()).total;
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

// B query rows; query row r reads cache batch row r / q_per_row
static int decode_impl(int phase, const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                       const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv, int64_t ckv_bstride,
                       int ckv_rstride, const mla_bf16_t* k_pe, int64_t kpe_bstride,
                       int kpe_rstride, int T, const int32_t* topk, int k,
                       const int32_t* end_pos, int B, int q_per_row, bool ragged, float scale,
                       mla_bf16_t* O, void* ws, size_t ws_bytes, int32_t* status,
                       void* stream) {
  if (phase < 0 || phase > 3 || (ragged && phase != 0)) return MLA_ERR_SHAPE;
  if (q_per_row < 1 || B % q_per_row != 0) return MLA_ERR_SHAPE;
  if (!q_nope || !q_pe || !wkv_b || !topk || !end_pos || !O) return MLA_ERR_NULL;
  if (int e = check_cache_args(c_kv, ckv_bstride, ckv_rstride, k_pe, kpe_bstride, kpe_rstride, T))
    return e;
  if (B < 1 || B > 65535 || k < 1 || k > 65536) return MLA_ERR_SHAPE;
  // the gather's 32-bit TMA row coordinate covers every cache row in use
  if ((long long)(B / q_per_row - 1) * (ckv_bstride / ckv_rstride) + T > 0x7fffffffLL)
    return MLA_ERR_SHAPE;
  if (!aligned16(q_nope) || !aligned16(q_pe) || !aligned16(wkv_b) || !aligned16(O))
    return MLA_ERR_ALIGN;
  if (!ws || !aligned256(ws)) return MLA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  const WsLayout L = ws_layout(B, max_clusters());
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  __nv_bfloat16* q_tilde = reinterpret_cast<__nv_bfloat16*>(wsb + L.q_tilde);
  __nv_bfloat16* opart = reinterpret_cast<__nv_bfloat16*>(wsb + L.opart);
  float* lse = reinterpret_cast<float*>(wsb + L.lse);
  __nv_bfloat16* omerged = reinterpret_cast<__nv_bfloat16*>(wsb + L.omerged);
  int32_t* cnt = reinterpret_cast<int32_t*>(wsb + L.cnt);
  int32_t* tstart = reinterpret_cast<int32_t*>(wsb + L.tstart);
  int32_t* tb = reinterpret_cast<int32_t*>(wsb + L.tb);
  int32_t* crow = reinterpret_cast<int32_t*>(wsb + L.crow);
  const core::Sched sch = ragged ? ragged_schedule_for(B, k, tstart, tb) : schedule_for(B, k);
  // whether any row can be split across clusters (ragged: decided on the device)
  const bool merge = ragged ? sch.nc > 1 : slots_of(sch, B) > 1;

  if (ragged) {
    // plain launches: they complete before the fold starts, so the attend
    // kernel (which may start during the fold) finds the tile counts
    row_tiles_kernel<<<(B + 7) / 8, 256, 0, st>>>(topk, k, B, cnt);
    if (int e = launch_status()) return e;
    tile_scan_kernel<<<1, 1024, 0, st>>>(cnt, B, sch.nc, tstart, tb, crow);
    if (int e = launch_status()) return e;
  }
  if (phase == 0 || phase == 1) {
    if (int e = launch_fold(reinterpret_cast<const __nv_bfloat16*>(q_nope),
                            reinterpret_cast<const __nv_bfloat16*>(wkv_b), q_tilde, B, status,
                            st))
      return e;
  }

  core::Params p;
  p.q_tilde = q_tilde;
  p.q_pe = reinterpret_cast<const __nv_bfloat16*>(q_pe);
  p.rows_per_b = ckv_bstride / ckv_rstride;
  p.q_per_row = q_per_row;
  p.T = T;
  p.topk = topk;
  p.k = k;
  p.end_pos = end_pos;
  p.B = B;
  p.sch = sch;
  p.crow = crow;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.opart = opart;
  p.lse = lse;
  p.omerged = omerged;
  p.status = status;
  if (phase == 0 || phase == 2) {
    alignas(64) CUtensorMap map_c, map_r;
    const unsigned long long rows =
        (unsigned long long)(B / q_per_row - 1) * p.rows_per_b + T;  // cache batch rows in use
    if (int e = make_row_map(&map_c, c_kv, kC, rows, ckv_rstride, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return e;
    if (int e = make_row_map(&map_r, k_pe, kR, rows, kpe_rstride, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return e;
    static std::atomic<unsigned long long> core_attr{0};
    if (int e = ensure_smem_attr(core_kernel, core::SMEM_BYTES, &core_attr)) return e;
    // In the full call the fold precedes it: programmatic serialisation lets
    // its set-up and first gathers (which read only the caller's inputs)
    // overlap the fold's tail.  Launched alone it waits for the stream.
    if (phase == 0) {
      if (int e = launch_pdl(core_kernel, dim3(2 * sch.nc), dim3(core::NTHREADS),
                             core::SMEM_BYTES, st, p, map_c, map_r))
        return e;
    } else {
      core_kernel<<<dim3(2 * sch.nc), core::NTHREADS, core::SMEM_BYTES, st>>>(p, map_c, map_r);
      if (int e = launch_status()) return e;
    }
  }
  if (phase == 0 || phase == 3) {
    if (merge) {
      const dim3 grid(sch.nc - 1, kH / 16);
      if (phase == 0) {
        if (int e = launch_pdl(combine_kernel, grid, dim3(256), 0, st, opart, lse, sch,
                               (const int32_t*)crow, omerged))
          return e;
      } else {
        combine_kernel<<<grid, 256, 0, st>>>(opart, lse, sch, crow, omerged);
        if (int e = launch_status()) return e;
      }
    }
    return launch_uv(reinterpret_cast<const __nv_bfloat16*>(wkv_b), omerged, B,
                     reinterpret_cast<__nv_bfloat16*>(O), status, st, phase == 0 || merge);
  }
  return MLA_OK;
}

extern "C" int mla_decode(const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                          const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv, int64_t ckv_bstride,
                          int ckv_rstride, const mla_bf16_t* k_pe, int64_t kpe_bstride,
                          int kpe_rstride, int T, const int32_t* topk, int k,
                          const int32_t* end_pos, int B, float scale, mla_bf16_t* O, void* ws,
                          size_t ws_bytes, int32_t* status, void* stream) {
  return decode_impl(0, q_nope, q_pe, wkv_b, c_kv, ckv_bstride, ckv_rstride, k_pe, kpe_bstride,
                     kpe_rstride, T, topk, k, end_pos, B, 1, false, scale, O, ws, ws_bytes, status,
                     stream);
}

extern "C" int mla_decode_mq(const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                             const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv, int64_t ckv_bstride,
                             int ckv_rstride, const mla_bf16_t* k_pe, int64_t kpe_bstride,
                             int kpe_rstride, int T, const int32_t* topk, int k,
                             const int32_t* end_pos, int B, int queries_per_row, float scale,
                             mla_bf16_t* O, void* ws, size_t ws_bytes, int32_t* status,
                             void* stream) {
  return decode_impl(0, q_nope, q_pe, wkv_b, c_kv, ckv_bstride, ckv_rstride, k_pe, kpe_bstride,
                     kpe_rstride, T, topk, k, end_pos, B, queries_per_row, true, scale, O, ws,
                     ws_bytes, status, stream);
}

extern "C" int mla_decode_phase(int phase, const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                                const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv,
                                int64_t ckv_bstride, int ckv_rstride, const mla_bf16_t* k_pe,
                                int64_t kpe_bstride, int kpe_rstride, int T, const int32_t* topk,
                                int k, const int32_t* end_pos, int B, float scale, mla_bf16_t* O,
                                void* ws, size_t ws_bytes, int32_t* status, void* stream) {
  return decode_impl(phase, q_nope, q_pe, wkv_b, c_kv, ckv_bstride, ckv_rstride, k_pe,
                     kpe_bstride, kpe_rstride, T, topk, k, end_pos, B, 1, false, scale, O, ws,
                     ws_bytes, status, stream);
}
