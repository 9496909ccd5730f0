/*
 * libshla -- absorbed sparse multi-head latent attention decode for B200
 * (sm_100a): the decode step of DeepSeek-V3.2-Exp's sparse latent attention,
 * with W_UK folded into the queries and W_UV applied after the latent mix.
 *
 * C ABI.  All tensor arguments are DEVICE pointers owned by the caller; the
 * library never allocates, frees or keeps per-call state, and it keeps no
 * pointer after a call returns.  Every compute entry point only enqueues work
 * on the given CUDA stream (``stream`` is a cudaStream_t; NULL = legacy
 * default stream) and returns at once.
 *
 * Element types:
 *   bf16  = 16-bit brain float, passed as raw bits (mla_bf16_t)
 *   fp32  = IEEE float
 *   int32 = int32_t
 * All arrays are row-major.  Unless a stride argument says otherwise, they are
 * contiguous.  Base pointers and row strides of every bf16/fp32 array must be
 * 16-byte aligned (MLA_ERR_ALIGN otherwise).
 *
 * Model dimensions are fixed ("Key heads" page, MLA init listing; "KV
 * compression" page):
 *   H  = 128 heads
 *   C  = 512 latent width (kv_lora_rank)
 *   R  = 64 shared rotary key width (qk_rope_head_dim)
 *   Dn = 128 non-rotary query/key width, Dv = 128 value width
 *   DIM = 7168 model width
 *
 * Return value: MLA_OK (0), or a negative MLA_ERR_* code for a synchronous
 * error found before anything was enqueued.  Asynchronous conditions go into
 * an optional caller-owned device int32 status[2]:
 *   status[0] |= MLA_STATUS_TIMEOUT  if a kernel gave up a bounded wait (the
 *                                    output is then undefined);
 *   status[1] += count of top-k entries that are neither -1 nor inside
 *                [0, min(end_pos[b], T)) (they are ignored).
 * The library never clears the status word.
 */
#ifndef SHLA_H_
#define SHLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t mla_bf16_t;

enum {
  MLA_OK = 0,
  MLA_ERR_NULL = -1,        /* a required pointer is NULL */
  MLA_ERR_SHAPE = -2,       /* a size or stride is out of range */
  MLA_ERR_ALIGN = -3,       /* a pointer or stride breaks 16-byte alignment */
  MLA_ERR_WORKSPACE = -4,   /* workspace pointer NULL or too small */
  MLA_ERR_UNSUPPORTED = -5, /* device is not sm_100 */
  MLA_ERR_CUDA = -6         /* a CUDA launch or attribute call failed */
};

#define MLA_STATUS_TIMEOUT 1

#define MLA_HEADS 128
#define MLA_LATENT 512
#define MLA_ROPE 64
#define MLA_NOPE 128
#define MLA_VDIM 128
#define MLA_ROW 576
#define MLA_DIM 7168

/* Human-readable text for a return code.  Static storage; never NULL. */
const char* mla_status_string(int code);

/*
 * Rotary embedding of feature pairs ("Rotated shared key" page,
 * the apply_rotary_emb code excerpt).
 *   x    bf16  [B, S, Hx, 64]
 *   rope fp32  [S, 32, 2]: (cos, sin) of the angle for sequence slot s and
 *              pair j; slot s of x uses row s (the caller offsets the table to
 *              the first position)
 *   interleaved != 0: pair j = (x[2j], x[2j+1]); result written back to
 *              (2j, 2j+1).  interleaved == 0: pair j = (x[j], x[j+32]); result
 *              written as all real parts then all imaginary parts.
 *   y    bf16  [B, S, Hx, 64]; may equal x (in place)
 * Rotation in fp32, one rounding to bf16.
 */
int mla_rope(const mla_bf16_t* x, const float* rope, int B, int S, int Hx, int interleaved,
             mla_bf16_t* y, void* stream);

/*
 * Cache write for new positions ("KV compression" page: the key-value
 * down-projection code excerpt, and its Explanation of the 576 values cached
 * per position):
 *   kv = x W_KVa (fp32 accumulation); latent = RMSNorm(kv[0:512]) * norm_w
 *   (y = v / sqrt(mean(v^2) + eps) * w, fp32); k_pe = interleaved RoPE of
 *   kv[512:576] at the row's position; both stored as bf16.
 *   x       bf16 [B, S, 7168]
 *   w_kva   bf16 [7168, 576]   (x W form: row i holds input feature i)
 *   norm_w  bf16 [512]
 *   rope    fp32 [S, 32, 2]    coefficients of positions start_pos .. start_pos+S-1
 *   c_kv    bf16 latent cache: element (b, t, c) at c_kv[b*ckv_bstride + t*ckv_rstride + c]
 *   k_pe    bf16 rotary cache: element (b, t, r) at k_pe[b*kpe_bstride + t*kpe_rstride + r]
 *           (fused [B, T, 576] rows: k_pe = c_kv + 512, both rstrides 576)
 *   T       cache capacity; requires 0 <= start_pos, start_pos + S <= T
 *   ws      device workspace of at least mla_cache_write_workspace_bytes(B*S)
 *           bytes, 256-byte aligned; contents need not be initialised
 * Requires 1 <= B*S <= 4096.
 * Two kernels are enqueued on `stream`: a split-K GEMM, then the finalize
 * kernel under programmatic dependent launch (it waits for the GEMM before
 * reading its partials).  For the caller nothing changes: work enqueued
 * after the call starts when the finalize kernel has finished.
 */
size_t mla_cache_write_workspace_bytes(int rows);
int mla_cache_write(const mla_bf16_t* x, const mla_bf16_t* w_kva, const mla_bf16_t* norm_w,
                    float eps, const float* rope, int B, int S, int start_pos,
                    mla_bf16_t* c_kv, int64_t ckv_bstride, int ckv_rstride,
                    mla_bf16_t* k_pe, int64_t kpe_bstride, int kpe_rstride, int T,
                    void* ws, size_t ws_bytes, void* stream);

/*
 * The cache write above without a workspace argument, for callers that
 * cannot allocate device memory when they call it: code running inside
 * callbacks of graph-based or embedding runtimes, decode loops whose runtime
 * forbids allocation after start-up, and hosts whose device memory belongs to
 * another allocator.  The pages describe no such variant; it exists only for
 * those callers.
 *
 * The split-K partial products go to one fixed device array inside this
 * library (MLA_NOALLOC_MAX_ROWS rows of partials, 4,128,768 bytes), which every
 * GPU that loads the library holds until the process exits.  Arguments,
 * layouts and results are those of mla_cache_write; B*S above
 * MLA_NOALLOC_MAX_ROWS returns MLA_ERR_SHAPE without touching the GPU.  The
 * function allocates nothing.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  The address belongs to the device's context: a call made after
 * the context was replaced (cudaDeviceReset and a new context) looks it up
 * again.  All calls share the array and it keeps the last call's contents;
 * every value a call reads from it is written earlier in the same call, so
 * nothing needs clearing, but calls that can overlap on the GPU (different
 * streams, or different host threads) race on it and must be serialised by
 * the caller.
 */
#define MLA_NOALLOC_MAX_ROWS 64
int mla_cache_write_noalloc(const mla_bf16_t* x, const mla_bf16_t* w_kva,
                            const mla_bf16_t* norm_w, float eps, const float* rope, int B, int S,
                            int start_pos, mla_bf16_t* c_kv, int64_t ckv_bstride,
                            int ckv_rstride, mla_bf16_t* k_pe, int64_t kpe_bstride,
                            int kpe_rstride, int T, void* stream);

/*
 * Absorbed sparse decode, one query per batch row ("Mix and project" page,
 * decode ("MQA decode") code excerpt):
 *   q~[b,h,:]  = q_nope[b,h,:] W_UK[h]            W_UK[h] = wkv_b[h, 0:128, :]
 *   s[b,h,t]   = (q~[b,h,:].c_KV[b,t,:] + q_pe[b,h,:].k_pe[b,t,:]) * scale
 *                for t in the selected set of row b
 *   A          = softmax_t(s)
 *   O~[b,h,:]  = sum_t A[b,h,t] c_KV[b,t,:]
 *   O[b,h,:]   = W_UV[h] O~[b,h,:]                W_UV[h] = wkv_b[h, 128:256, :]
 * The selected keys of row b are the entries of topk[b, :] inside
 * [0, min(end_pos[b], T)); -1 entries are padding.  Other entries are
 * ignored and counted in status[1].  A row with no valid entry gets O = 0.
 * The pages' index mask is a set (a position listed twice is selected once);
 * this call does not look for repeats: each valid entry is one key, so a
 * position listed twice counts twice.  Callers pass distinct positions (an
 * indexer's top-k does), and then the two agree.
 *   q_nope  bf16 [B, 128, 128]
 *   q_pe    bf16 [B, 128, 64]   (already rotated)
 *   wkv_b   bf16 [128, 256, 512] ([out, in] storage of the 512 -> 128*256 projection)
 *   c_kv, k_pe, strides, T: cache as in mla_cache_write (read only)
 *   topk    int32 [B, k]   positions, in any order; distinct (see above)
 *   end_pos int32 [B]
 *   scale   softmax scale (192^-0.5 * mscale^2 in the model)
 *   O       bf16 [B, 128, 128]
 *   ws      device workspace of at least mla_decode_workspace_bytes(B, k) bytes,
 *           256-byte aligned; contents need not be initialised
 *   status  optional int32[2] (see top of file), may be NULL
 * Requires 1 <= B <= 65535 and 1 <= k <= 65536.
 *
 * Arithmetic: the scores are accumulated in fp32 by the tensor cores (each CTA
 * of a pair over half of the 576 columns; the two fp32 partial sums are added
 * in fp32), then scaled, masked, maximised, shifted by the running maximum
 * and exponentiated in fp32; row sums, the output accumulator and the
 * rescaling are fp32.  Rounded to bf16, as tensor-core operands: q~ (the
 * fold's output), the softmax weights P = 2^(s - m) (at most 2^8: the running
 * maximum is raised once a tile's maximum exceeds it by more than 8 log2
 * units), and the per-split partial outputs that the merge reads.  O is
 * rounded to bf16 once, at the end.
 *
 * Work split: the flattened list of (row, 64-key tile) is cut into equal
 * contiguous ranges, one per SM pair; a row cut between two ranges is merged
 * from their partial results by log-sum-exp.  The ranges depend on the
 * number of SM pairs the device runs the kernel on, so on devices with
 * different SM counts the split rows (and the last bits of their outputs)
 * may differ; on one device the result is the same on every call.
 *
 * The call enqueues three or four kernels on `stream`.  The first waits for
 * the stream's earlier work as usual.  The later ones use programmatic
 * dependent launch: each may start its set-up while its predecessor drains,
 * and reads that predecessor's results only once it has finished.  For the
 * caller nothing changes: work enqueued after the call starts when the call's
 * last kernel has finished, and the inputs must not be modified before then.
 */
size_t mla_decode_workspace_bytes(int B, int k);
int mla_decode(const mla_bf16_t* q_nope, const mla_bf16_t* q_pe, const mla_bf16_t* wkv_b,
               const mla_bf16_t* c_kv, int64_t ckv_bstride, int ckv_rstride,
               const mla_bf16_t* k_pe, int64_t kpe_bstride, int kpe_rstride, int T,
               const int32_t* topk, int k, const int32_t* end_pos, int B, float scale,
               mla_bf16_t* O, void* ws, size_t ws_bytes, int32_t* status, void* stream);

/*
 * Several query rows per cache batch row: query row r (0 <= r < B) reads
 * cache batch row r / queries_per_row, with its own q_nope[r], q_pe[r],
 * topk[r, :] and end_pos[r]; everything else is mla_decode's definition
 * (mla_decode is the case queries_per_row = 1).  Two uses:
 *
 *   multi-query decode: S new tokens of one sequence scored in one step
 *   (speculative or multi-token-prediction tokens); row b * S + s holds token
 *   s of sequence b, end_pos[b * S + s] its causal limit.
 *
 *   sparse prefill ("Mix and project" page, the MHA prefill branch of the
 *   forward excerpt, with the index mask added to the causal mask): a prompt
 *   of S tokens of sequence b, cached at positions 0 .. S-1, gives rows
 *   b * S + s with end_pos = s + 1.  The prefill branch expands per-head keys
 *   k = [c_KV W_UK[h] ; k_pe] and values c_KV W_UV[h] and scores every prompt
 *   position under the mask; folding W_UK into the query and W_UV after the
 *   mix gives the same result in exact arithmetic ("Key heads" page), and
 *   only the selected positions are read.  Entries past the causal limit are
 *   excluded as the mask excludes them (and counted in status[1] like any
 *   entry outside [0, end_pos)); pass -1 for them to keep the count clean.
 *
 *   q_nope, q_pe, topk, end_pos, O: B query rows, layouts as mla_decode
 *   c_kv, k_pe, strides, T: B / queries_per_row cache batch rows
 *   ws: mla_decode_workspace_bytes(B, k) bytes
 *
 * Ragged lists: the lists of prefill tokens and new tokens end in -1 padding
 * of different lengths.  Two small kernels run first: one counts, per query
 * row, the 64-entry tiles up to the last one that holds an entry other than
 * -1 (at least one), and one prefix-sums the counts and cuts the work into
 * ranges that balance the tiles plus a fixed cost per row; the tiles after a
 * row's last listed entry are not run.  The split points therefore differ
 * from mla_decode's, and with one query per row the two calls agree within
 * rounding, not bit for bit.
 * Requires queries_per_row >= 1 dividing B, and every cache row in use
 * addressable as a 32-bit row index: (B / queries_per_row - 1) *
 * (ckv_bstride / ckv_rstride) + T <= 2^31 - 1 (else MLA_ERR_SHAPE).
 */
int mla_decode_mq(const mla_bf16_t* q_nope, const mla_bf16_t* q_pe, const mla_bf16_t* wkv_b,
                  const mla_bf16_t* c_kv, int64_t ckv_bstride, int ckv_rstride,
                  const mla_bf16_t* k_pe, int64_t kpe_bstride, int kpe_rstride, int T,
                  const int32_t* topk, int k, const int32_t* end_pos, int B, int queries_per_row,
                  float scale, mla_bf16_t* O, void* ws, size_t ws_bytes, int32_t* status,
                  void* stream);

/*
 * The same call split into its three phases, for timing one of them alone:
 *   phase 1: fold of W_UK into the queries (writes q~ into ws)
 *   phase 2: gather + scores + softmax + latent mix (reads q~; writes the
 *            mixed latent O~ of each row held by one cluster, and the
 *            partial O~ and log-sum-exp of each segment of a split row, into ws)
 *   phase 3: log-sum-exp merge of the split rows (one launch, skipped when no
 *            row is split), then O = O~ W_UV^T (reads ws, writes O)
 *   phase 0: all three (identical to mla_decode)
 * Phases must run in order on one stream with the same arguments and
 * workspace; each phase alone leaves O undefined until phase 3 has run.
 */
int mla_decode_phase(int phase, const mla_bf16_t* q_nope, const mla_bf16_t* q_pe,
                     const mla_bf16_t* wkv_b, const mla_bf16_t* c_kv, int64_t ckv_bstride,
                     int ckv_rstride, const mla_bf16_t* k_pe, int64_t kpe_bstride,
                     int kpe_rstride, int T, const int32_t* topk, int k, const int32_t* end_pos,
                     int B, float scale, mla_bf16_t* O, void* ws, size_t ws_bytes,
                     int32_t* status, void* stream);

/*
 * Fold of W_UK into the queries, the first step of mla_decode ("Mix and
 * project" page, decode branch: einsum bshd,hdc->bshc):
 *   q_tilde[b,h,c] = sum_d q_nope[b,h,d] wkv_b[h,d,c]     bf16 [B, 128, 512]
 * fp32 accumulation, one rounding to bf16.  Requires 1 <= B <= 65535.
 */
int mla_fold_wuk(const mla_bf16_t* q_nope, const mla_bf16_t* wkv_b, int B,
                 mla_bf16_t* q_tilde, void* stream);

/*
 * Test hook: the decode index mask ("Mix and project" page, decode branch:
 * a -inf row over [0, end_pos) with the indexer's positions scattered to 0).
 *   mask uint8 [B, T]: 1 where t is listed in topk[b] and t < end_pos[b], else 0.
 * Invalid entries are counted in status[1] (status may be NULL).
 */
int mla_index_mask(const int32_t* topk, int B, int k, const int32_t* end_pos, int T,
                   uint8_t* mask, int32_t* status, void* stream);

/*
 * Test hook: the row gather of mla_decode.  rows[b, j, :] = the 576 cached
 * values (latent then rotary key) of position topk[b, j], or zeros when the
 * entry is -1 or invalid (invalid ones are counted in status[1]).
 *   rows bf16 [B, k, 576]
 */
int mla_gather_rows(const mla_bf16_t* c_kv, int64_t ckv_bstride, int ckv_rstride,
                    const mla_bf16_t* k_pe, int64_t kpe_bstride, int kpe_rstride, int T,
                    const int32_t* topk, int B, int k, const int32_t* end_pos,
                    mla_bf16_t* rows, int32_t* status, void* stream);

/*
 * Test hook: the expiry path of the bounded waits.  Every wait in the
 * library's kernels (mbarrier phases, the MMA issuer's event loop) gives up
 * after 1 s, sets MLA_STATUS_TIMEOUT in status[0] and lets its kernel wind
 * down, so that a lost arrival ends as an error the host can read instead of
 * a hung GPU.  This call launches one block of two warps that wait, through
 * the same code, on an mbarrier that nothing arrives on; it returns after the
 * limit with status[0] |= MLA_STATUS_TIMEOUT and gave_up[0] += 2 (one per
 * warp).  The GPU context stays usable.
 *   status  int32[2] device (status[1] untouched); gave_up int32[1] device
 */
int mla_wait_limit_check(int32_t* status, int32_t* gave_up, void* stream);

/* The most ranges (SM pairs) that share one row in mla_decode's work split
 * for (B, k) on the current device (1: no row is split). */
int mla_decode_num_splits(int B, int k);

/*
 * Output projection of the attention block ("Mix and project" page: the
 * output projection wo, the only step that mixes heads, 16,384 x 7,168
 * weights; the decode excerpt applies it as wo(x.flatten(2))):
 *   Delta[b, n] = sum over h, d of O[b, h, d] W_O[n, h * 128 + d]
 *     O      bf16 [B, 128, 128]   (the mla_decode output; flattened head-major)
 *     w_o    bf16 [7168, 16384]   ([out, in] storage)
 *     delta  bf16 [B, 7168]
 * fp32 accumulation.  A row tile of W_O whose K range is split between CTAs
 * is summed from fp32 partials in a fixed order, so the result is the same
 * on every run.  Requires 1 <= B <= 65535 and a caller-owned device
 * workspace of at least mla_out_proj_workspace_bytes(B) bytes, 256-byte
 * aligned (MLA_ERR_WORKSPACE otherwise).  status may be NULL (see above).
 * Two kernels are enqueued; the second uses programmatic dependent launch
 * (as described for mla_decode), with the same stream semantics for the
 * caller.
 */
size_t mla_out_proj_workspace_bytes(int B);
int mla_out_proj(const mla_bf16_t* O, const mla_bf16_t* w_o, int B, mla_bf16_t* delta, void* ws,
                 size_t ws_bytes, int32_t* status, void* stream);

/*
 * Query path ("Query rotary up-projection" page: the MLA init and forward
 * excerpts; W_QR is output features 128-191 of each head's 192 in wq_b):
 *   qr[b, :]   = RMSNorm(x[b] wq_a^T) * q_norm_w   (fp32 norm, qr rounded to bf16)
 *   q[b, h, :] = (qr[b] wq_b^T)[192 h .. 192 h + 191]
 *   q_nope[b, h, :] = q[b, h, 0:128]
 *   q_pe[b, h, :]   = interleaved rotation of q[b, h, 128:192] by rope[pos[b]]
 *     x        bf16 [B, 7168]
 *     wq_a     bf16 [1536, 7168]       ([out, in])
 *     q_norm_w bf16 [1536], eps >= 0   (RMSNorm y = x / sqrt(mean(x^2) + eps) * w)
 *     wq_b     bf16 [24576, 1536]      ([out, in], 128 heads x (128 + 64))
 *     rope     fp32 [T, 32, 2]         ((cos, sin) per position and pair)
 *     pos      int32 [B]               (the query position of each row)
 *     q_nope   bf16 [B, 128, 128], q_pe bf16 [B, 128, 64]: the mla_decode inputs
 * A row whose pos is outside [0, T) gets q_pe = 0 and is counted in
 * status[1].  Partials are summed in a fixed order (results identical on
 * every run).  Requires 1 <= B <= 65535 and a device workspace of at least
 * mla_query_proj_workspace_bytes(B) bytes, 256-byte aligned.  Four kernels
 * are enqueued; the last three use programmatic dependent launch (as
 * described for mla_decode), with the same stream semantics for the caller.
 */
size_t mla_query_proj_workspace_bytes(int B);
int mla_query_proj(const mla_bf16_t* x, const mla_bf16_t* wq_a, const mla_bf16_t* q_norm_w,
                   float eps, const mla_bf16_t* wq_b, const float* rope, int T,
                   const int32_t* pos, int B, mla_bf16_t* q_nope, mla_bf16_t* q_pe, void* ws,
                   size_t ws_bytes, int32_t* status, void* stream);

/*
 * Test hook (host only, no device call): the work split of the
 * weight-streaming GEMM behind mla_out_proj and mla_query_proj for a
 * [n_out, k_in] weight.  Row tile m (128 weight rows) and K chunk j (128
 * columns) form unit m * nch + j; CTA c of a batch block takes units
 * [c * tot / nc, (c + 1) * tot / nc).  Writes plan[0..3] = tot, nc, nch,
 * slots, and for every row tile m first_last[2m], first_last[2m + 1] = the
 * first and last CTA holding a unit of tile m (the partial of CTA c for tile
 * m goes to slot c - first); first_last may be NULL.  Requires
 * n_out % 128 == 0 and k_in % 128 == 0, both positive (else MLA_ERR_SHAPE).
 */
int mla_xwt_plan(int n_out, int k_in, int32_t* plan, int32_t* first_last);

#ifdef __cplusplus
}
#endif

#endif /* SHLA_H_ */
