/*
 * pa.h — C ABI of libpa: causal GQA prefill attention of a query chunk against a long
 * history held in a paged KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (what the pages describe; they give no formula, this is the plain reading):
 *   "Metal: paged-KV prefill is 4.43x slower than contiguous KV at 32K" (BaseRT issue #51),
 *   sections "Results" and "Scaling characteristic": prefill attention of a chunk whose
 *   K/V are read through a paged cache, which must cost about what a contiguous cache costs.
 *   "perf: scale prefill attention splits with GPU cores on Apple7/8" (splash PR #33),
 *   section "What changed": the history of a piece is cut into splits so that short pieces
 *   at long history fill the GPU; a reduce merges the split partials; the planner picks the
 *   split count and workspace from the core count, KV heads and piece tiles.
 *
 *   For chunk row i (absolute position H+i) and Q head h, with G = Hq/Hkv and g = floor(h/G):
 *     key j (0 <= j <= H+i) is  k_pool[page_table[j / PS]][j % PS][g][:]  (v likewise)
 *     out[i][h][:] = sum_j softmax_j(scale * q[i][h][:] . K[j][:]) * V[j][:]
 *   with scale = 1/sqrt(D) unless given. The chunk's own K/V (positions H..H+R-1) must
 *   already be in the cache.
 *
 * Threading and memory: every function is reentrant. The library never allocates, frees or
 * synchronises device memory in pa_prefill / pa_combine; the caller owns every buffer. All
 * device work is enqueued on the caller's stream (a cudaStream_t passed as pa_stream_t).
 * Status codes are returned; nothing throws across the ABI.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same representation as cudaStream_t / CUstream (NULL = the legacy default stream). */
typedef struct CUstream_st* pa_stream_t;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, inconsistent sizes, plan mismatch */
  PA_ERR_UNSUPPORTED = -2,  /* shape outside the supported set (see pa_plan) */
  PA_ERR_WORKSPACE = -3,    /* lse_ws missing or smaller than plan->ws_bytes */
  PA_ERR_CUDA = -4,         /* a CUDA runtime/driver call failed (launch, tensor map, ...) */
  PA_ERR_TIMEOUT = -5,      /* a kernel wait gave up (reported by pa_device_error) */
  PA_ERR_PAGE_INDEX = -6    /* a page-table entry was outside [0, num_pages) */
} pa_status;

/* Split policies for pa_plan (how the history of a piece is partitioned). */
typedef enum {
  /* B200: the schedule that minimises the simulated makespan of the launch on num_sms SMs
   * (items are dispatched in order to the first free SM), plus the combine's HBM cost: a
   * uniform split count (units longest first), or the balanced schedule when it is faster. */
  PA_POLICY_MAKESPAN = 0,
  /* The rule of splash PR #33 ("What changed"): min(256, max(32, 32*cores/kv_heads)) /
   * tiles, clamped to 1..32, with cores = num_sms and tiles = Q tiles per KV head. */
  PA_POLICY_CORES = 1,
  /* The earlier rule quoted in splash PR #33: clamp(32 / tiles, 1, 32), with tiles taken as
   * the threadgroups over all KV heads (the reading under which every listed piece got 1). */
  PA_POLICY_LEGACY = 2,
  /* B200: cut the history of some row blocks at arbitrary KV tiles so that every SM (or SM
   * pair) gets the same number of KV tiles: the row blocks' tiles are laid end to end and cut
   * where each worker's equal share ends (McNaughton's wrap-around rule), no piece shorter
   * than a few tiles. Uncut row blocks write `out` directly; the parts of a cut one are merged
   * by pa_combine. Falls back to the makespan policy's uniform splits only when the
   * schedule would not fit the kernel's tables (512 items, 256 cut row blocks, 32 parts);
   * the plan's `policy` field says which was used. */
  PA_POLICY_BALANCED = 3
} pa_policy;

/* Rows of the packed (token, head) Q tile, and keys per KV tile, of the kernel. */
#define PA_TILE_ROWS 128
#define PA_TILE_KEYS 128
#define PA_MAX_SPLITS 32

/*
 * A launch plan. Filled by pa_plan; callers read it and pass it back unchanged.
 *
 * Q rows are packed as (token, head-in-group) pairs with the head index fastest: packed row
 * r of KV head g is token r / G, Q head g*G + r % G. A Q tile is PA_TILE_ROWS consecutive
 * packed rows (a tile may start inside a token's head group). Work units are
 * (KV head, Q tile, split); split s of a tile whose tokens end at t_last covers KV tiles
 * [s*n/S, (s+1)*n/S) of the n = ceil((H + t_last + 1) / PA_TILE_KEYS) tiles it sees. With
 * ctas_per_unit = 2 a unit is a pair of consecutive Q tiles (2t, 2t+1) on a CTA pair, and t_last
 * is that of the pair's last tile.
 *
 * Plans with policy == PA_POLICY_BALANCED use work items instead of uniform splits. A row
 * block is (unit of ctas_per_unit Q tiles, KV head), numbered rb = (q_units-1-u)*Hkv + g with
 * q_units = ceil(q_tiles / ctas_per_unit) (last unit first); an item is a run [kt0, kt1) of
 * the KV tiles its unit sees; `units` counts the items and `splits` is the largest number of
 * items of one row block. pa_schedule_items lists them.
 */
typedef struct {
  int32_t num_sms;        /* SMs the plan was made for */
  int32_t n_q_heads;      /* Hq */
  int32_t n_kv_heads;     /* Hkv (Hq % Hkv == 0) */
  int32_t head_dim;       /* D: 64, 128 or 256 */
  int32_t page_size;      /* PS: power of two, 16..128 (ignored when paged == 0) */
  int32_t group;          /* G = Hq / Hkv */
  int32_t chunk_rows;     /* R: query rows of the piece (>= 1) */
  int32_t q_tiles;        /* ceil(R * G / PA_TILE_ROWS) per KV head */
  int32_t splits;         /* S: 1..PA_MAX_SPLITS (balanced: most items of one row block) */
  int32_t paged;          /* 1: k/v are page pools read through page_table; 0: contiguous */
  int32_t dtype;          /* pa_dtype of q, k, v */
  int32_t policy;         /* pa_policy used (or -1 when splits was overridden); balanced
                           * plans read PA_POLICY_BALANCED whichever policy chose them */
  int32_t ctas_per_unit;  /* 2: head_dim 256 runs on CTA pairs (two Q tiles per unit); else 1 */
  int32_t batch;          /* decode plans (pa_decode_plan): sequences; prefill plans: 0 */
  int64_t hist_len;       /* H: keys in the cache before the piece */
  int64_t units;          /* Hkv * ceil(q_tiles / ctas_per_unit) * S units (CTAs or pairs);
                           * balanced: the number of items */
  float scale;            /* softmax scale actually used */
  float est_us;           /* the planner's time estimate for prefill + combine (microseconds) */
  uint64_t ws_bytes;      /* bytes of lse_ws needed: S*R*Hq*(D+1)*4 if S > 1, else 0;
                           * balanced: slots * ctas_per_unit*128 * (D+1) * 4, one slot per
                           * item of a cut row block */
} pa_plan_t;

/*
 * pa_plan — choose the split count and workspace for one piece.
 *   num_sms          SMs of the device (148 on B200); > 0.
 *   n_q_heads, n_kv_heads, head_dim, page_size, chunk_rows, hist_len, dtype: the piece.
 *   scale            softmax scale; 0 selects 1/sqrt(head_dim).
 *   splits_override  0: the policy decides; 1..32: use exactly this split count.
 *   policy           a pa_policy (used when splits_override == 0).
 *   paged            1: K/V through a page table; 0: contiguous [H+R][Hkv][D].
 *   plan             out: the plan (host memory owned by the caller).
 * Returns PA_OK, PA_ERR_INVALID_ARG or PA_ERR_UNSUPPORTED. Pure host code; no CUDA calls.
 * Source: splash PR #33 "What changed" (split count from cores, KV heads and tiles; the
 * workspace is sized by the planner).
 */
int pa_plan(int num_sms, int n_q_heads, int n_kv_heads, int head_dim, int page_size,
            int chunk_rows, int64_t hist_len, int dtype, float scale, int splits_override,
            int policy, int paged, pa_plan_t* plan);

/*
 * pa_schedule_items — the work items of a balanced plan, in launch order: for item i,
 * items[4i..4i+3] = (rb, kt0, kt1, slot), slot = -1 for an uncut row block (written to out)
 * or the workspace slot of its partial. Writes at most `cap` items (items may be NULL).
 * Returns the number of items, 0 for a plan that is not balanced, or PA_ERR_INVALID_ARG when
 * the plan does not match its own schedule. Pure host code.
 */
int pa_schedule_items(const pa_plan_t* plan, int32_t* items, int cap);

/*
 * pa_prefill — split-KV prefill attention of one piece, enqueued on `stream`.
 *   q            device, [R][Hq][D] of dtype, contiguous, 16-byte aligned.
 *   k_pool,v_pool device, paged: [num_pages][PS][Hkv][D]; contiguous: [H+R][Hkv][D]; dtype,
 *                contiguous, 16-byte aligned. Pool slots that hold no key may hold any bits
 *                (NaN included); they never reach the output.
 *   page_table   device int32 [ceil((H+R)/PS)]: logical page -> physical page (paged only;
 *                may be NULL when paged == 0). An entry outside [0, num_pages) reads zeros
 *                and raises PA_ERR_PAGE_INDEX in pa_device_error.
 *   num_pages    pages in each pool (paged only).
 *   hist_len, chunk_rows: must equal the plan's.
 *   out          device fp32 [R][Hq][D]. Written when plan->splits == 1; balanced plans
 *                write the rows of uncut row blocks here.
 *   lse_ws       device fp32 workspace of ws_bytes >= plan->ws_bytes (used when S > 1):
 *                partial outputs O_s [S][R][Hq][D] (each normalised over its split), then
 *                base-2 log-sum-exp of the scaled scores lse_s [S][R][Hq] (-inf: no key).
 *                Balanced plans: O [slots][rows][D] then lse [slots][rows], rows =
 *                ctas_per_unit*128 packed rows of the item's row block.
 * When S > 1 (or the plan is balanced with a cut row block), call pa_combine afterwards on
 * the same stream to produce `out`.
 * Returns PA_OK or an error status; launch errors are PA_ERR_CUDA. Device-side conditions
 * (bad page entry, wait timeout) are reported by pa_device_error.
 */
int pa_prefill(const pa_plan_t* plan, const void* q, const void* k_pool, const void* v_pool,
               const int32_t* page_table, int64_t num_pages, int64_t hist_len, int chunk_rows,
               float* out, float* lse_ws, uint64_t ws_bytes, pa_stream_t stream);

/*
 * pa_combine — log-sum-exp merge of the S split partials in lse_ws into out (fp32
 * [R][Hq][D]): out = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M), M = max_s lse_s.
 * No-op returning PA_OK when plan->splits == 1. For balanced plans it merges the parts of
 * each cut row block into that block's rows of out. Source: splash PR #33, the prefill
 * attention "reduce" that merges the split partials (decode-profile tables).
 */
int pa_combine(const pa_plan_t* plan, const float* lse_ws, uint64_t ws_bytes, float* out,
               pa_stream_t stream);

/*
 * pa_decode_plan — plan batched paged decode attention: `batch` sequences, one new query token
 * each (its own K/V already in the pool), every key of the sequence visible. Fills a plan whose
 * chunk_rows = batch (one row per sequence), q_tiles = 1 (needs G <= 128), batch = batch and
 * splits S: the history of every sequence is cut into S splits so that batch * Hkv * S units
 * fill the CTA slots (about two units per slot, at most 32 and at most the 128-key tiles of
 * max_seq_len), or exactly splits_override. A slot is an SM, or half an SM when the group
 * G <= 8 and D is 128 or 256 (those steps run two CTAs per SM; see pa_decode). ws_bytes = S * batch * Hq * (D + 1) * 4 when S > 1,
 * in the layout of pa_prefill's split workspace with batch in place of R, so pa_combine
 * merges it. Returns PA_OK, PA_ERR_INVALID_ARG or PA_ERR_UNSUPPORTED. Pure host code.
 * Source: generation over a long cache, where every new token reads its sequence's whole
 * window (llama.cpp PR #27977, "qwen4exp: reduce the generation slowdown as context grows",
 * description), on the same paged cache the prefill fills (BaseRT issue #51, "Serving impact":
 * continuous batching implies the paged cache).
 */
int pa_decode_plan(int num_sms, int n_q_heads, int n_kv_heads, int head_dim, int page_size,
                   int batch, int64_t max_seq_len, int dtype, float scale, int splits_override,
                   pa_plan_t* plan);

/*
 * pa_decode — batched paged decode attention on `stream`. With G <= 8 at head dim 128 or 256 the
 * keys take the tensor cores' M side (S^T = K Q^T, O^T = V^T P^T, two CTAs per SM); otherwise
 * the single-CTA prefill kernel runs one 128-row Q tile per unit.
 *   q            device [batch][Hq][D] of dtype: the new token of each sequence.
 *   k_pool,v_pool device [num_pages][PS][Hkv][D], 16-byte aligned.
 *   block_table  device int32 [batch][table_stride]: sequence b's logical page -> physical page.
 *   seq_lens     device int32 [batch]: keys of sequence b (its new token included), 0..
 *                table_stride * PS. A sequence with no key gets zeros. A length outside that
 *                range is clamped into it and reported as PA_ERR_PAGE_INDEX by pa_device_error.
 *   out          device fp32 [batch][Hq][D]. Written when plan->splits == 1.
 *   lse_ws       workspace of plan->ws_bytes when S > 1; then call pa_combine (same plan).
 * Returns PA_OK, PA_ERR_INVALID_ARG, PA_ERR_WORKSPACE or PA_ERR_CUDA; bad page entries and
 * wait timeouts are reported by pa_device_error.
 * The kernel reads seq_lens first and starts the units of the longest sequences first, so the
 * short ones fill the end of the launch: for batch <= 256 by exact length (ties in sequence
 * order), for larger batches by length class floor(log2(ceil(len / 128))) (sequence order
 * within a class). The order changes timing only, never the results.
 */
int pa_decode(const pa_plan_t* plan, const void* q, const void* k_pool, const void* v_pool,
              const int32_t* block_table, int table_stride, const int32_t* seq_lens,
              int64_t num_pages, float* out, float* lse_ws, uint64_t ws_bytes,
              pa_stream_t stream);

/*
 * Batched prefill (continuous batching): several sequences in one launch, each a chunk of
 * q_lens[b] query rows at its own history of hist_lens[b] keys, all on one page pool. The
 * causal rule is the single-piece one, per sequence: row i of sequence b sees keys
 * 0 .. hist_lens[b] + i of that sequence. A decode step is the case q_lens[b] = 1,
 * hist_lens[b] = keys before the new token. Source: the pages' chunked prefill (BaseRT issue
 * #51, "Results"; splash PR #33, "What changed") applied to every sequence of a batch; the
 * batching itself is the serving engine's, which the pages do not describe.
 *
 * pa_batch_plan — the balanced schedule of the batch (host only): the row blocks of all
 * sequences, longest first, cut by the wrap-around rule into at most 512 items on num_sms SMs
 * (when the cuts would not fit in 512 items, every row block is one item, longest first).
 *   q_lens     host int32 [batch], >= 0 (a sequence with 0 rows has no output rows).
 *   hist_lens  host int64 [batch], >= 0.
 *   batch      1 .. 256 sequences; at most 512 row blocks in all ((KV head, 128-row Q tile
 *              unit) pairs: Hkv * ceil(ceil(q_lens[b] * G / 128) / ctas_per_unit) summed).
 * Fills a plan with batch = batch, chunk_rows = sum of q_lens, hist_len = the largest history,
 * policy = PA_POLICY_BALANCED, units = items, splits = the most items of one row block, and
 * ws_bytes = slots * ctas_per_unit*128 * (D + 1) * 4. The arrays are not kept: pass the same
 * ones to pa_batch_prefill and pa_batch_combine, which rebuild the schedule from them.
 * Returns PA_OK, PA_ERR_INVALID_ARG or PA_ERR_UNSUPPORTED (too many sequences or row blocks).
 */
int pa_batch_plan(int num_sms, int n_q_heads, int n_kv_heads, int head_dim, int page_size,
                  int batch, const int32_t* q_lens, const int64_t* hist_lens, int dtype,
                  float scale, pa_plan_t* plan);

/*
 * pa_batch_prefill — batched prefill attention on `stream`.
 *   q            device [sum q_lens][Hq][D] of dtype: the sequences' chunks, packed in order.
 *   k_pool,v_pool device [num_pages][PS][Hkv][D]; the chunks' own K/V already in place.
 *   block_table  device int32 [batch][table_stride]: sequence b's logical page -> physical page;
 *                entries past ceil((hist_lens[b] + q_lens[b]) / PS) are not read.
 *   out          device fp32 [sum q_lens][Hq][D]; rows of uncut row blocks are written here.
 *   lse_ws       workspace of plan->ws_bytes when ws_bytes > 0; then call pa_batch_combine.
 * Returns PA_OK, PA_ERR_INVALID_ARG (arrays that do not rebuild the plan's schedule, or a
 * plan that is not a batch plan), PA_ERR_WORKSPACE or PA_ERR_CUDA.
 * A batch in which every sequence has at most one query row, with G <= 8 at head dim 128 or
 * 256, runs on pa_decode's kernel (keys on the tensor cores' M side, two CTAs per SM), and
 * pa_batch_plan cuts its items for two CTA slots per SM.
 */
int pa_batch_prefill(const pa_plan_t* plan, const int32_t* q_lens, const int64_t* hist_lens,
                     const void* q, const void* k_pool, const void* v_pool,
                     const int32_t* block_table, int table_stride, int64_t num_pages, float* out,
                     float* lse_ws, uint64_t ws_bytes, pa_stream_t stream);

/* pa_batch_schedule_items — the work items of a batch plan, as pa_schedule_items lists them;
 * rb is a global row block: sequence b owns rb0_b .. rb0_b + its row blocks - 1, with rb0_b
 * the row blocks of sequences 0 .. b-1, numbered within the sequence like a single piece's. */
int pa_batch_schedule_items(const pa_plan_t* plan, const int32_t* q_lens,
                            const int64_t* hist_lens, int32_t* items, int cap);

/* pa_batch_combine — merge the partials of the cut row blocks into out (no-op when none). */
int pa_batch_combine(const pa_plan_t* plan, const int32_t* q_lens, const int64_t* hist_lens,
                     const float* lse_ws, uint64_t ws_bytes, float* out, pa_stream_t stream);

/* Bytes of the device-resident scratch used by pa_prefill_noalloc (64 MiB). */
#define PA_NOALLOC_WS_BYTES (64ull << 20)

/*
 * pa_prefill_noalloc — pa_prefill followed by pa_combine, for callers that cannot allocate
 * device memory: for example a plugin inside a serving engine that has reserved all device
 * memory for its KV-cache pool and exposes no allocator, or a caller that cannot afford the
 * implicit device synchronisation an allocation may cause. (The pages describe no such entry
 * point; it has no counterpart there.)
 *   Arguments are those of pa_prefill, without lse_ws / ws_bytes: when plan->splits > 1 the
 *   split partials go to a scratch array that the library holds in device memory on every
 *   device it is loaded on (PA_NOALLOC_WS_BYTES, kept until the process exits). out is
 *   written in full, as pa_prefill + pa_combine would write it.
 *   The first call on a device looks the scratch's device address up (a runtime call, made
 *   with that device current); make that first call before any stream capture. The address
 *   is kept for the life of the process: a device reset (cudaDeviceReset) or a teardown of
 *   the device's primary context after that first call is not supported.
 *   Every call shares the one scratch array, which keeps the last call's contents (nothing in
 *   it needs to start at zero: each call writes every entry it reads). Calls whose work may
 *   overlap on the GPU (different streams, or several host threads without ordering) race on
 *   it: order them, e.g. issue them on one stream.
 * Returns PA_ERR_WORKSPACE when plan->ws_bytes exceeds PA_NOALLOC_WS_BYTES, else what
 * pa_prefill / pa_combine return. Allocates nothing (no cudaMalloc, no cudaFree).
 */
int pa_prefill_noalloc(const pa_plan_t* plan, const void* q, const void* k_pool,
                       const void* v_pool, const int32_t* page_table, int64_t num_pages,
                       int64_t hist_len, int chunk_rows, float* out, pa_stream_t stream);

/*
 * pa_kv_append — write a chunk's new K and V rows into the paged pools through the page table,
 * enqueued on `stream`: the step before pa_prefill (BaseRT issue #51, "Results": the chunk's
 * K/V are published to pages and prefill reads every key, its own included, through the table).
 *   k_new, v_new   device [R][Hkv][D] of dtype, contiguous, 16-byte aligned.
 *   k_pool, v_pool device [num_pages][PS][Hkv][D] (as pa_prefill), 16-byte aligned.
 *   page_table     device int32 [ceil((H+R)/PS)]; hist_len H: position of the first new row;
 *                  chunk_rows R (0: nothing to do).
 * Row i goes to page page_table[(H+i)/PS], slot (H+i)%PS, all Hkv heads at once; nothing else
 * in the pools changes. An entry outside [0, num_pages) skips its rows and raises
 * PA_ERR_PAGE_INDEX in pa_device_error. Returns PA_OK, PA_ERR_INVALID_ARG,
 * PA_ERR_UNSUPPORTED (head_dim not 64/128/256, page_size not a power of two in 16..128) or
 * PA_ERR_CUDA.
 */
int pa_kv_append(int n_kv_heads, int head_dim, int page_size, int dtype, const void* k_new,
                 const void* v_new, void* k_pool, void* v_pool, const int32_t* page_table,
                 int64_t num_pages, int64_t hist_len, int chunk_rows, pa_stream_t stream);

/*
 * pa_kv_publish — the page publish of the contiguous-staging route (BaseRT issue #51,
 * "Expected vs actual": bulk prefill on a contiguous staging buffer, completed K/V then
 * published to pages). Copies staged rows [first_pos, first_pos + rows) of
 * k_staged / v_staged (device [T][Hkv][D], the prompt's positions from 0) to their pages:
 * position p goes to page page_table[p/PS], slot p%PS. Same kernel, checks and errors as
 * pa_kv_append (whose k_new is the staged buffer advanced by first_pos rows).
 */
int pa_kv_publish(int n_kv_heads, int head_dim, int page_size, int dtype, const void* k_staged,
                  const void* v_staged, void* k_pool, void* v_pool, const int32_t* page_table,
                  int64_t num_pages, int64_t first_pos, int rows, pa_stream_t stream);

/*
 * pa_device_error — synchronise the current device, then read (and with reset != 0,
 * clear) the library's device-side error word. *flags receives its bits
 * (1: page index out of range, 2: a wait timed out). Returns PA_OK when no bit is set,
 * PA_ERR_PAGE_INDEX or PA_ERR_TIMEOUT for the first set bit, PA_ERR_CUDA on failure.
 */
int pa_device_error(int* flags, int reset);

/* pa_set_wait_timeout_ns — upper bound of every kernel-side wait (default 2e9 ns). A wait
 * that exceeds it makes the kernel set the timeout bit, stop its work and exit. */
void pa_set_wait_timeout_ns(uint64_t ns);

/*
 * pa_selftest_timeout — enqueue a one-warp kernel that waits on a barrier nothing ever
 * completes, with a wait limit of timeout_ns; the wait gives up, sets the timeout bit and
 * the kernel exits. Lets tests check the timeout path without hanging a GPU.
 */
int pa_selftest_timeout(uint64_t timeout_ns, pa_stream_t stream);

/* pa_status_string — static description of a status code. */
const char* pa_status_string(int status);

/*
 * pa_pieces — cut a chunk of chunk_rows query rows at history hist_len into pieces the way the
 * pages' engine does at long context (splash PR #33, "What changed": 512 rows from 32K history,
 * 256 from 64K, 128 past about 128K, per rows * (history + rows) <= 2^25): each piece is the
 * largest power of two r of the rows left with r * (history + r) <= 2^log2_budget (at least one
 * row), and each piece's history includes the pieces before it. Writes at most `cap` piece sizes
 * (rows_out may be NULL) and returns the number of pieces, or PA_ERR_INVALID_ARG. Pure host code.
 * On B200 the balanced planner fills the GPU without cutting chunks; the rule is kept to
 * reproduce the pages' pieces (the 32K-history workload of four 512-row pieces).
 */
int pa_pieces(int chunk_rows, int64_t hist_len, int log2_budget, int32_t* rows_out, int cap);

/* pa_cores_policy_splits — the split rule of splash PR #33 ("What changed") for a GPU with
 * `cores` cores, `kv_heads` KV heads and `tiles` tiles per KV head. Pure host function. */
int pa_cores_policy_splits(int cores, int kv_heads, int tiles);

/* pa_legacy_policy_splits — the earlier rule clamp(32 / tiles, 1, 32) quoted there, with
 * tiles = threadgroups over all KV heads. Pure host function. */
int pa_legacy_policy_splits(int kv_heads, int tiles);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
