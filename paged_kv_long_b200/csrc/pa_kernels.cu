// pa_kernels.cu — sm_100a kernels of libpa and their C-ABI entry points.
//
// prefill_kernel: one CTA per unit — (KV head, packed Q tile, history split) for uniform splits,
//   a work item (a run of a row block's KV tiles) for balanced plans, (sequence, KV head, split)
//   for batched decode whose group the swapped decode kernel does not take.
//   The operation is prefill attention of a query chunk against a long history read through
//   a paged KV cache (BaseRT issue #51, "Results"), with the history of a piece cut into
//   splits whose partials a reduce merges (splash PR #33, "What changed"). The B200 design:
//   * warps 5-7 (copy warps) read the page table and issue TMA boxes into a ring of 16 KB,
//     128-byte-swizzled shared-memory panels: K as one box per (page, 64-wide D panel), V as
//     boxes of up to one page covering all of D;
//   * warp 4 (MMA; one lane) issues tcgen05.mma: S = Q K^T into one of two tensor-memory S
//     buffers (Q and K from shared memory), then O += P V with P read from tensor memory where
//     the softmax wrote it over its own S buffer (fp32 accumulation in tensor memory);
//   * warps 0-3 (softmax, one thread per packed Q row = tensor-memory lane) load the GQA-
//     packed Q tile, read S with tcgen05.ld, apply the causal mask by select, keep the
//     running max and sum (rescaling O only when the max grows by more than 2^8), write P
//     (rounded to the input type) to tensor memory, and finally write O / l (fp32) or the
//     split partial and its base-2 log-sum-exp.
//   Every wait is bounded: on expiry the kernel sets the timeout bit, abandons its work,
//   waits for its own copies and MMAs in flight, frees tensor memory and exits.
// prefill_pair_kernel (prefill_pair.cuh): head dim 256 on CTA pairs (cta_group::2, M = 256).
// decode_kernel, decode_batch_kernel (decode_kernel.cuh): one query token per sequence with the
//   keys on the MMA's M side (S^T = K Q^T, O^T = V^T P^T), two CTAs per SM.
// combine_kernel: one warp per (row, head) merges the S partials with a log-sum-exp
//   weighting (the "reduce" of splash PR #33); combine_blocks_kernel does the same for the
//   cut row blocks of balanced plans.
// kv_append_kernel (kv_append.cuh): a chunk's K/V rows into their pages.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <cstring>
#include <atomic>
#include <mutex>

#include "pa.h"
#include "pa_geometry.h"
#include "pa_schedule.h"
#include "sm100.cuh"

namespace pa {

__device__ unsigned int g_pa_error_flags;
constexpr unsigned kFlagPage = 1u;
constexpr unsigned kFlagTimeout = 2u;

constexpr int kPanel = 128 * 128;          // bytes of one 128-row x 128-byte panel (a slot)
constexpr int kThreads = 256;  // 4 softmax warps, 1 MMA warp, 3 TMA-issuing warps
constexpr int kIssuers = 3;    // TMA issue latency is per issuing warp: three overlap it
constexpr int kMmaWarp = 4;
constexpr float kRescaleLog2 = 8.0f;       // rescale O only when the max grows by > 2^8
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0;              // O accumulator: columns [0, D)
constexpr uint32_t kSCol0 = 256;           // S buffers: [256, 384) and [384, 512)
constexpr uint32_t kPColOff = 64;          // P (16-bit pairs) over the upper half of its S

struct PrefillArgs {
  const uint16_t* q;
  const int32_t* page_table;
  float* out;
  float* ws_o;
  float* ws_lse;
  int64_t hist_len;
  int64_t table_len;
  int64_t total_keys;
  int32_t R, Hq, Hkv, G;
  int32_t q_tiles, splits;
  int32_t page_rows;     // key rows per page: the page size, or kTileKeys when contiguous
  int32_t page_shift;    // log2(page_rows)
  int32_t pages_per_tile;
  int32_t k_rows;        // key rows per K box (CTA-pair kernel: <= 64, half a tile)
  int32_t v_rows;        // key rows per V box (<= page_rows; a box is at most one slot)
  int32_t v_shift;       // log2(v_rows)
  int32_t num_pages;
  int32_t oob_row;       // a key-row coordinate past the pool: the TMA fills zeros there
  float scale_log2;      // softmax scale * log2(e)
  uint64_t timeout_ns;
  int32_t q_tma;           // 1: the Q tile arrives by tensor copy (CTA-pair kernel, G | 128)
  int32_t k_atoms;         // 1: a K box is 8 keys x all 4 panels (CTA-pair kernel, pages of 16)
  int64_t ws_split_rows;   // workspace rows of one split: R * Hq (decode: batch * Hq)
  // Batched decode (batch > 0, single-CTA kernel): unit u is (sequence u / (Hkv*S), KV head,
  // split); sequence b has seq_lens[b] keys, its page-table row at page_table + b * table_stride,
  // its one query token at q + b*Hq*D and its output rows at out + b*Hq*D.
  int32_t batch;
  int32_t table_stride;
  const int32_t* seq_lens;
  int32_t balanced;        // 1: CTA (pair) b runs work item b of the item table
  int32_t rows_per_block;  // packed rows of a row block (balanced workspace slots)
  // Batched prefill (balanced and batch > 0): an item's row block names its sequence (the item
  // table's sequence list); q_row0 is that sequence's first row in the packed Q / out arrays.
  int32_t q_row0;
};

// The work items of a balanced plan, passed by value (kernel parameter space): no device
// allocation, and a CUDA graph that captures the launch keeps its own copy.
struct ItemTable {
  PaItem item[kMaxItems];
  PaSeq seq[kMaxSeqs];  // batched plans: the sequences, rb0 ascending
};
// SoftmaxCtx::slot value of the uniform-split schedule (destination from the split index).
constexpr int kSlotUniform = -2;

// Batched plans: point the arguments at the sequence that owns global row block rb (its Q and
// output rows, its page-table row, its history and rows) and return the row block's number
// within the sequence.
template <int D>
__device__ __forceinline__ int32_t batch_rebase(PrefillArgs& a, const ItemTable& t, int32_t rb) {
  const int b = seq_of_rb(t.seq, a.batch, rb);
  const PaSeq sq = t.seq[b];
  a.q += (int64_t)sq.q_row0 * a.Hq * D;
  a.out += (int64_t)sq.q_row0 * a.Hq * D;
  a.page_table += (int64_t)b * a.table_stride;
  a.hist_len = sq.hist;
  a.R = sq.rows;
  a.total_keys = (int64_t)sq.hist + sq.rows;
  a.table_len = (a.total_keys + a.page_rows - 1) / a.page_rows;
  a.q_tiles = (int32_t)q_tiles_for(sq.rows, a.G);
  a.q_row0 = sq.q_row0;
  return rb - sq.rb0;
}

// Device-length decode: block r·Hkv·S .. of the grid runs the sequence of rank r, where the rank
// orders the sequences by length, longest first (ties by index). The block scheduler hands out
// blocks in index order as SMs free up, so the units of the longest sequences start first and
// the short ones fill the end (longest-processing-time-first list scheduling). A bijection of
// 0 .. B-1 whatever the lengths hold. Every thread of the block takes part (two block barriers);
// `scratch` is B + 1 words of shared memory that no copy writes yet.
constexpr int kRankedSeqsMax = 256;  // longer batches: by length class (seq_of_class_rank)

__device__ __noinline__ int seq_of_rank(const int32_t* lens, int B, int r, int32_t* scratch) {
  for (int i = threadIdx.x; i < B; i += blockDim.x) scratch[i] = __ldg(lens + i);
  if (threadIdx.x == 0) scratch[B] = r;
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int32_t lb = scratch[b];
    int rank = 0;
    for (int c = 0; c < B; ++c) {
      const int32_t lc = scratch[c];
      rank += (lc > lb) | ((lc == lb) & (c < b));
    }
    if (rank == r) scratch[B] = b;  // exactly one b has rank r
  }
  __syncthreads();
  return scratch[B];
}

// Longer batches: the same longest-first rule at the granularity of a factor of two. Sequences
// are ordered by length class floor(log2(KV tiles)) (a sequence with no key counts as one
// tile), the longest class first, sequence order within a class; O(B / threads) per block.
// The class of rank r comes from per-class counts; its member of index r - (the counts of the
// longer classes) from a block scan of per-thread counts over contiguous runs of sequences.
// A bijection of 0 .. B-1. Every thread of the block takes part (five block barriers);
// `scratch` is 67 words of shared memory that no copy writes yet.
__device__ __forceinline__ int len_class(int32_t len) {
  const int tiles = len <= 0 ? 1 : (int)(((int64_t)len + kTileKeys - 1) / kTileKeys);
  return 31 - __clz(tiles);
}

__device__ __noinline__ int seq_of_class_rank(const int32_t* lens, int B, int r,
                                              int32_t* scratch) {
  const int t = threadIdx.x, nt = blockDim.x, lane = t & 31, wid = t >> 5;
  int32_t* cnt = scratch;               // [32] sequences per class
  int32_t* wsum = scratch + 32;         // [32] per-warp totals of the scan
  int32_t* res = scratch + 64;          // [2] class of rank r, rank within that class
  int32_t* found = scratch + 66;        // [1] the sequence
  if (t < 32) cnt[t] = 0;
  __syncthreads();
  for (int b = t; b < B; b += nt) atomicAdd(&cnt[len_class(__ldg(lens + b))], 1);
  __syncthreads();
  if (t == 0) {
    int acc = 0, c = 31;
    while (c > 0 && r >= acc + cnt[c]) acc += cnt[c--];  // r < B: stops at the class holding r
    res[0] = c;
    res[1] = r - acc;
    found[0] = -1;
  }
  __syncthreads();
  const int C = res[0], want = res[1];
  const int per = (B + nt - 1) / nt;
  const int b0 = min(B, t * per), b1 = min(B, b0 + per);
  int mine = 0;
  for (int b = b0; b < b1; ++b) mine += len_class(__ldg(lens + b)) == C;
  int incl = mine;  // inclusive scan of the per-thread counts in thread order
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < wid; ++w) before += wsum[w];
  const int start = before + incl - mine;  // class-C members in the runs before this thread's
  if (want >= start && want < start + mine) {
    int k = want - start;
    for (int b = b0; b < b1; ++b)
      if (len_class(__ldg(lens + b)) == C && k-- == 0) {
        found[0] = b;
        break;
      }
  }
  __syncthreads();
  return found[0];
}

// Shared-memory layout. The ring holds 16 KB slots, filled and consumed in the order K0, K1,
// V0, K2, V1, ..., V_{n-1}; every K or V tile takes NP consecutive slots (mod NSLOT). A K
// tile is one 64-wide D panel per slot (128 keys x 128 B, the K-major B operand of Q K^T),
// loaded as one TMA box per (page, panel). A V tile is a run of TMA boxes of v_rows keys x
// all NP panels (each box panel-major, the MN-major B operand of P V); a box never straddles
// two slots. Fill number q is issued by TMA warp q % kIssuers.
// SQ (small Q): every Q tile of the launch holds at most 8 packed rows (decode: one token of
// G <= 8 heads). Q then takes one 8-row swizzle atom per panel (1 KB, not 16 KB) and the
// A operand of Q K^T repeats that atom over the 128 rows of the MMA (descriptor stride 0):
// rows 8..127 of S are copies of rows 0..7, which belong to no output. The freed 60 KB
// deepen the ring to 13 slots, so the copies run further ahead of a unit that is bound by
// its K/V reads.
template <int D, bool SQ = false>
struct Cfg {
  static constexpr int NP = D / 64;                  // 64-element panels per K/V/Q row
  static constexpr int NSLOT = SQ ? 13 : (D == 256) ? 10 : 12;  // ring of 16 KB slots
  static constexpr int Q_PANEL = SQ ? 1024 : kPanel; // bytes of one Q panel
  static constexpr int Q_SBO = SQ ? 0 : 1024;        // Q descriptor: bytes between 8-row atoms
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = Q_OFF + NP * Q_PANEL;
  static constexpr int BAR_OFF = RING_OFF + NSLOT * kPanel;
  // barriers: full[NSLOT], empty[NSLOT], q_full, s_full[2], p_full[2], pv_done[2], mma_done
  static constexpr int B_FULL = 0, B_EMPTY = NSLOT, B_QFULL = 2 * NSLOT, B_SFULL = 2 * NSLOT + 1,
                       B_PFULL = 2 * NSLOT + 3, B_PVDONE = 2 * NSLOT + 5,
                       B_MMADONE = 2 * NSLOT + 7, N_BARS = 2 * NSLOT + 8;
  static constexpr int MISC_OFF = BAR_OFF + 8 * N_BARS;
  static constexpr int SMEM = MISC_OFF + 16;
  static constexpr int LAUNCH_SMEM = SMEM + 1024;    // slack to align the base to 1024 B
  static constexpr int PANEL_LOG = (NP == 4) ? 9 : (NP == 2) ? 8 : 7;  // log2(NP * 128)
  static_assert(LAUNCH_SMEM <= 232448, "exceeds 227 KB of shared memory per CTA");
};

// Position of tile j's V in the load order K0, K1, V0, K2, V1, ..., V_{n-1}.
__device__ __forceinline__ uint32_t v_item(int j, int n) {
  return j == n - 1 ? 2u * n - 1u : 2u * j + 2u;
}

// Byte offset, inside a V tile, of (key row k of the tile, panel p).
template <int NP, int PANEL_LOG>
__device__ __forceinline__ uint32_t v_offset(uint32_t k, uint32_t p, int v_shift) {
  return ((k >> v_shift) << (v_shift + PANEL_LOG)) + ((p << v_shift) << 7) +
         ((k & ((1u << v_shift) - 1u)) << 7);
}

// ---------------------------------------------------------------- bounded waits
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       uint64_t timeout_ns, bool honour_abort) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (honour_abort && *abort_flag) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        *abort_flag = 1;
        atomicOr(&g_pa_error_flags, kFlagTimeout);
        return false;
      }
    }
  }
}

// One thread waits (the single-lane roles).
__device__ __forceinline__ bool thread_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            uint64_t timeout_ns) {
  return mbar_try_wait(bar, parity) || wait_slow(bar, parity, abort_flag, timeout_ns, true);
}

// All 32 lanes wait; the result is uniform across the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns) {
  bool ok = mbar_try_wait(bar, parity) || wait_slow(bar, parity, abort_flag, timeout_ns, true);
  return __all_sync(0xffffffffu, ok);
}

// Teardown wait: ignores the abort flag (copies and MMAs in flight always finish), bounded.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint64_t timeout_ns) {
  if (!mbar_try_wait(bar, parity)) wait_slow(bar, parity, abort_flag, timeout_ns, false);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if constexpr (BF16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

// Softmax + epilogue warps (warps 0-3: one thread per packed Q row = tensor-memory lane), for
// both kernels. The pair kernel's second CTA announces Q and P on the first CTA's barriers
// (remote arrivals); everything else it reads and writes is its own.
struct SoftmaxCtx {
  uint32_t sb, q_off;
  uint32_t bar_sfull, bar_pvdone;      // local barriers: S buffers 0/1, PV groups of even/odd tiles
  uint32_t arrive_qfull, arrive_pfull; // where Q / P readiness is announced (maybe remote)
  bool remote_arrive;
  uint32_t tmem;
  int64_t qt;
  int g, s;
  int64_t kt0;
  int n;
  int slot;       // workspace slot of a balanced item's partial, -1: final output,
                  // kSlotUniform: uniform splits (out when S == 1, else split s's partial)
  int row0;       // first packed row of this CTA inside its row block (balanced slots)
  uint32_t stage_off;  // shared memory free once the last PV is done: 128 x (4D + 16) bytes
  volatile int* abort_flag;
  uint64_t tmo;
};

// Epilogue of one softmax thread (packed row r of its CTA's Q tile, tensor-memory lane
// t_lane): O / l from tensor memory to the output row, or to the workspace row of a partial
// together with its base-2 log-sum-exp. The row goes through shared memory (x.stage_off, idle
// once the last P V is done; rows 16 bytes apart from a multiple of 128 so that a warp's
// stores spread over the banks) and leaves as one contiguous bulk copy.
template <int D>
__device__ __forceinline__ void write_row(const PrefillArgs& a, const SoftmaxCtx& x, int r,
                                          bool valid, int64_t tok, int head, float m_run,
                                          float l_run, uint32_t t_lane) {
  const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
  int64_t ws_row = -1;  // workspace row of a partial; -1: the final output
  if (x.slot >= 0)
    ws_row = (int64_t)x.slot * a.rows_per_block + x.row0 + r;
  else if (x.slot == kSlotUniform && a.splits > 1)
    ws_row = (int64_t)x.s * a.ws_split_rows + tok * a.Hq + head;
  float* dst = ws_row < 0 ? a.out + (tok * a.Hq + head) * (int64_t)D : a.ws_o + ws_row * D;
  const uint32_t srow = x.sb + x.stage_off + (uint32_t)r * (uint32_t)(D * 4 + 16);
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    float o[32];
    tmem_ld32(t_lane + kOCol + 32u * c, o);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 8; ++i)
      st_shared_v4(srow + 128u * c + 16u * i, __float_as_uint(o[4 * i] * inv_l),
                   __float_as_uint(o[4 * i + 1] * inv_l), __float_as_uint(o[4 * i + 2] * inv_l),
                   __float_as_uint(o[4 * i + 3] * inv_l));
  }
  fence_proxy_async_smem();
  if (valid) bulk_store(dst, srow, D * 4);
  bulk_commit();
  bulk_wait_read_all();
  if (valid && ws_row >= 0) a.ws_lse[ws_row] = l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
}

template <int D, bool PAGED, bool BF16, bool SQ, class VTail>
__device__ __forceinline__ void softmax_role(const PrefillArgs& a, const SoftmaxCtx& x,
                                             VTail&& v_tail) {
  constexpr int NP = D / 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sb = x.sb, tmem = x.tmem;
  const int64_t qt = x.qt, kt0 = x.kt0;
  const int g = x.g, n = x.n;
  volatile int* abort_flag = x.abort_flag;
  const uint64_t tmo = x.tmo;
  auto arrive = [&](uint32_t addr) {
    if (x.remote_arrive)
      mbar_arrive_remote(addr);
    else
      mbar_arrive(addr);
  };
  {
    const int r = threadIdx.x;  // packed Q row = tensor-memory lane
    const int64_t grow = qt * kTileRows + r;
    const int64_t tok = grow / a.G;
    const bool valid = tok < a.R;
    const int head = g * a.G + (int)(grow % a.G);
    if (!a.q_tma) {
      // Q tile -> shared memory as K-major rows of 64-element panels, 128-byte swizzle (when
      // the tensor copy cannot: it loads whole tokens, so it needs G to divide 128). Small Q:
      // rows 0..7 only, one 1 KB atom per panel.
      constexpr uint32_t kQPanel = SQ ? 1024u : (uint32_t)kPanel;
      const uint4* src =
          reinterpret_cast<const uint4*>(a.q + (valid ? (tok * a.Hq + head) * (int64_t)D : 0));
      if (!SQ || r < 8) {
#pragma unroll
        for (int p = 0; p < NP; ++p) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = valid ? __ldg(src + p * 8 + c) : make_uint4(0u, 0u, 0u, 0u);
            st_shared_v4(sb + x.q_off + p * kQPanel + r * 128 + ((c ^ (r & 7)) << 4), v.x, v.y,
                         v.z, v.w);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) arrive(x.arrive_qfull);
    }

    const int64_t limit = valid ? a.hist_len + tok : -1;  // last key this row may see
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
    float m_run = -INFINITY;  // running max of scale*log2(e)*score
    float l_run = 0.f;        // running sum of the probabilities (fp32)
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sbuf = j & 1;
      const uint32_t s_col = kSCol0 + 128u * sbuf;
      const int64_t key0 = (kt0 + j) * kTileKeys;
      if (!warp_wait(x.bar_sfull + 8u * sbuf, (j >> 1) & 1, abort_flag, tmo)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kTileKeys];
#pragma unroll
      for (int c = 0; c < kTileKeys / 32; ++c)
        tmem_ld32(t_lane + s_col + 32u * c, *reinterpret_cast<float(*)[32]>(&sv[32 * c]));
      tmem_wait_ld();

      // causal mask by select (masked scores become -inf, whatever bits they held)
      const int64_t rel64 = limit - key0;
      if (rel64 < kTileKeys - 1) {
        const int rel = rel64 < -1 ? -1 : (int)rel64;
#pragma unroll
        for (int c = 0; c < kTileKeys; ++c)
          if (c > rel) sv[c] = -INFINITY;
      }
      // row max: eight independent chains, then a tree
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = sv[i];
#pragma unroll
      for (int c = 8; c < kTileKeys; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_new = fmaxf(m_run, mx * a.scale_log2);
      const bool need = m_new > m_run + kRescaleLog2;
      // PV of tile i completes phase i/2 of pv_done[i % 2]. Parity waits are sound only if no
      // phase is skipped: the softmax observes PV_{j-2} before it releases P_j (PV_j, the next
      // completion on that barrier, cannot happen earlier), and PV_{j-1} only when O must be
      // rescaled. P_j thus never waits for the PV just before it.
      if (j == 0) {
        if (need) m_run = m_new;
      } else if (__any_sync(0xffffffffu, need)) {
        // O must not change under a running MMA: wait for PV of the previous tile.
        if (!warp_wait(x.bar_pvdone + 8u * ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, tmo)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float f = need ? ex2(m_run - m_new) : 1.0f;
        l_run *= f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(t_lane + kOCol + 32u * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tmem_st32(t_lane + kOCol + 32u * c, o);
        }
        tmem_wait_st();
        if (need) m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      const float2 nm2 = make_float2(-m_use, -m_use);
      float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // two 64-key halves -> 32 columns of P each
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float2 x = ffma2(make_float2(sv[64 * h + c], sv[64 * h + c + 1]), sc2, nm2);
          const float2 pr = make_float2(ex2(x.x), ex2(x.y));
          ls[(c >> 1) & 3] = fadd2(ls[(c >> 1) & 3], pr);
          pk[c >> 1] = pack2<BF16>(pr.x, pr.y);
        }
        tmem_st32u(t_lane + s_col + kPColOff + 32u * h, pk);
      }
      l_run += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y) + (ls[2].x + ls[2].y) +
               (ls[3].x + ls[3].y);
      if (j >= 2 && !warp_wait(x.bar_pvdone + 8u * (j & 1), ((j - 2) >> 1) & 1, abort_flag, tmo)) {
        ok = false;
        break;
      }

      if constexpr (PAGED) {
        if (key0 + kTileKeys > a.total_keys) {
          const bool zero_me = key0 + r >= a.total_keys;
          if (!v_tail(j, zero_me ? r : -1)) {
            ok = false;
            break;
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      // P lives in tensor memory: a CTA-scope release orders it (see mbar_arrive_remote_tc);
      // a tile whose V rows this thread zeroed in shared memory takes the cluster-scope one.
      if (lane == 0) {
        if (x.remote_arrive && !(PAGED && key0 + kTileKeys > a.total_keys))
          mbar_arrive_remote_tc(x.arrive_pfull + 8u * sbuf);
        else
          arrive(x.arrive_pfull + 8u * sbuf);
      }
    }

    if (ok && n >= 2)
      ok = warp_wait(x.bar_pvdone + 8u * ((n - 2) & 1), ((n - 2) >> 1) & 1, abort_flag, tmo);
    if (ok) ok = warp_wait(x.bar_pvdone + 8u * ((n - 1) & 1), ((n - 1) >> 1) & 1, abort_flag, tmo);
    if (ok) {
      tc_fence_after();
      write_row<D>(a, x, r, valid, tok, head, m_run, l_run, t_lane);
    }
  }
}

// Key-row coordinate in the pool of page `lane` (< pages per tile) of KV tile kt0 + jt of a
// unit with n tiles: page_table[page] << page_shift, or oob_row (the TMA fills zeros there)
// past the unit or the table; an entry outside the pool is reported (by `report` lanes) and
// read as oob_row. Contiguous K/V: the tile's first key row.
template <bool PAGED>
__device__ __forceinline__ int32_t tile_page_row(const PrefillArgs& a, int64_t kt0, int n,
                                                 int jt, int lane, bool report) {
  int32_t row = a.oob_row;
  if constexpr (PAGED) {
    const int64_t lp = (kt0 + jt) * a.pages_per_tile + lane;
    if (jt < n && lane < a.pages_per_tile && lp < a.table_len) {
      const int32_t e = __ldg(a.page_table + lp);
      if (e >= 0 && e < a.num_pages)
        row = e << a.page_shift;
      else if (report)
        atomicOr(&g_pa_error_flags, kFlagPage);
    }
  } else {
    row = (int32_t)((kt0 + jt) * kTileKeys);
  }
  return row;
}

// Device-length decode, block blockIdx.x: unit (sequence of rank blockIdx.x / (Hkv·S), KV head
// g, split s) over its keys 0 .. len-1 (the new token's own included, all visible). Points a at
// the sequence (Q, output and workspace rows, page-table row, lengths) and gives the unit's KV
// tiles [kt0, kt1). A length outside 0 .. the table row's keys is reported like a bad page
// entry and clamped. Every thread of the block takes part (block barriers in the ranking);
// `scratch`: shared memory that no copy writes yet (see seq_of_rank).
template <int D>
__device__ __forceinline__ void decode_unit(PrefillArgs& a, int32_t* scratch, int* g, int* s,
                                            int64_t* kt0, int64_t* kt1) {
  const int64_t per_seq = (int64_t)a.Hkv * a.splits;
  const int64_t rem = blockIdx.x % per_seq;
  int64_t b = blockIdx.x / per_seq;
  b = a.batch <= kRankedSeqsMax ? seq_of_rank(a.seq_lens, a.batch, (int)b, scratch)
                                : seq_of_class_rank(a.seq_lens, a.batch, (int)b, scratch);
  *g = (int)(rem / a.splits);
  *s = (int)(rem % a.splits);
  int64_t len = __ldg(a.seq_lens + b);
  const int64_t cap = (int64_t)a.table_stride * a.page_rows;  // keys the table row can map
  if (len < 0 || len > cap) {
    if (threadIdx.x == 0 && *g == 0 && *s == 0) atomicOr(&g_pa_error_flags, kFlagPage);
    len = len < 0 ? 0 : cap;
  }
  a.q += b * a.Hq * D;
  a.out += b * a.Hq * D;
  if (a.ws_o) {
    a.ws_o += b * a.Hq * D;
    a.ws_lse += b * a.Hq;
  }
  a.page_table += b * a.table_stride;
  a.hist_len = len > 0 ? len - 1 : 0;
  a.total_keys = len;
  a.table_len = (len + a.page_rows - 1) / a.page_rows;
  a.R = len > 0 ? 1 : 0;
  split_range((len + kTileKeys - 1) / kTileKeys, *s, a.splits, kt0, kt1);
}

// A unit without KV tiles (a split past its tile's keys, or a decode sequence with no key):
// zeros for the output (one split) or an empty partial (zeros, LSE -inf), by threads < 128.
template <int D>
__device__ __forceinline__ void empty_unit(const PrefillArgs& a, int64_t qt, int g, int s) {
  if (threadIdx.x >= kTileRows) return;
  const int64_t grow = qt * kTileRows + threadIdx.x;
  const int64_t tok = grow / a.G;
  if (tok >= (a.batch > 0 ? 1 : a.R)) return;
  const int head = g * a.G + (int)(grow % a.G);
  if (a.splits == 1) {
    float4* d4 = reinterpret_cast<float4*>(a.out + (tok * a.Hq + head) * D);
    for (int i = 0; i < D / 4; ++i) d4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    const int64_t row = (int64_t)s * a.ws_split_rows + tok * a.Hq + head;
    float4* d4 = reinterpret_cast<float4*>(a.ws_o + row * D);
    for (int i = 0; i < D / 4; ++i) d4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    a.ws_lse[row] = -INFINITY;
  }
}

// The copy warps of the single-CTA kernels (warp w of kIssuers): fill the ring of NSLOT 16 KB
// slots at `ring` in the order K0, K1, V0, K2, V1, ..., V_{n-1} (see Cfg) for the n KV tiles
// kt0 .. kt0 + n - 1 of KV head g, fill number q by warp q % kIssuers. full[i] / empty[i] are the slots'
// barriers (8 bytes apart). pre_row0 / pre_row1: lane i's page row of tiles 0 / 1 (read
// before the set-up). Every copy has landed when this returns.
template <int NP, int NSLOT, int PANEL_LOG, bool PAGED>
__device__ __forceinline__ void kv_copy_role(const PrefillArgs& a, const CUtensorMap* tm_k,
                                             const CUtensorMap* tm_v, int g, int64_t kt0, int n,
                                             int w, uint32_t ring, uint32_t bar_full, uint32_t bar_empty,
                                             int32_t pre_row0, int32_t pre_row1,
                                             volatile int* abort_flag, uint64_t tmo) {
  const int lane = threadIdx.x & 31;
  auto slot_addr = [&](uint32_t slot) -> uint32_t { return ring + slot * kPanel; };
  auto full = [&](uint32_t slot) -> uint32_t { return bar_full + 8u * slot; };
  const int ppt = a.pages_per_tile;   // pages per KV tile (1 when contiguous)
  const int prow = a.page_rows;       // key rows per page (kTileKeys when contiguous)
  const int vsub = prow >> a.v_shift; // V boxes per page
  const int vbytes_log = a.v_shift + PANEL_LOG;   // log2 of a V box's bytes
  const int vbox_per_slot = 1 << (14 - vbytes_log);
  bool ok = true;
  // Lane i < ppt holds the key-row coordinate of page i of a tile (read one tile ahead).
  auto fetch = [&](int jt) -> int32_t {
    int32_t row = a.oob_row;
    if constexpr (PAGED) {
      const int64_t lp = (kt0 + jt) * ppt + lane;
      if (jt < n && lane < ppt && lp < a.table_len) {
        const int32_t e = __ldg(a.page_table + lp);
        if (e >= 0 && e < a.num_pages)
          row = e << a.page_shift;
        else if (w == 0)
          atomicOr(&g_pa_error_flags, kFlagPage);
      }
    } else {
      row = (int32_t)((kt0 + jt) * kTileKeys);
    }
    return row;
  };
  // Wait until fill q's slot is free and announce its bytes; false if the wait gave up.
  auto acquire = [&](uint32_t q) -> bool {
    const uint32_t slot = q % NSLOT;
    bool r_ok = q < (uint32_t)NSLOT ||
                warp_wait(bar_empty + 8u * slot, ((q / NSLOT) - 1) & 1, abort_flag, tmo);
    if (r_ok && lane == 0) mbar_arrive_expect_tx(full(slot), kPanel);
    __syncwarp();
    return r_ok;
  };
  int32_t row_prev = a.oob_row, row_cur = pre_row0, row_next = pre_row1;
  uint32_t issued_end = 0;  // one past the last fill number this warp issued
  for (int j = 0; j <= n && ok; ++j) {
    if (j < n) {  // K tile j: panel k in fill q, one box per page (lane i: page i)
      const uint32_t item = j == 0 ? 0u : 2u * j - 1u;
      for (int k = 0; k < NP && ok; ++k) {
        const uint32_t q = item * NP + k;
        if ((int)(q % kIssuers) != w) continue;
        if (!(ok = acquire(q))) break;
        const uint32_t slot = q % NSLOT;
        if (lane < ppt)
          tma_load_3d(slot_addr(slot) + lane * prow * 128, tm_k, full(slot), k * 64, g,
                      row_cur);
        issued_end = q + 1;
      }
    }
    if (ok && j >= 1) {  // V tile j-1: slot k holds boxes k*vbox_per_slot + lane
      const uint32_t item = v_item(j - 1, n);
      for (int k = 0; k < NP && ok; ++k) {
        const uint32_t q = item * NP + k;
        if ((int)(q % kIssuers) != w) continue;
        if (!(ok = acquire(q))) break;
        const uint32_t slot = q % NSLOT;
        const int b = k * vbox_per_slot + lane;        // box index inside the V tile
        const int pg = b / vsub, sub = b - pg * vsub;  // its page and place in the page
        const int32_t prow_b = __shfl_sync(0xffffffffu, row_prev, pg & 31);
        if (lane < vbox_per_slot)
          tma_load_4d(slot_addr(slot) + (lane << vbytes_log), tm_v, full(slot), 0,
                      prow_b + (sub << a.v_shift), 0, g);
        issued_end = q + 1;
      }
    }
    row_prev = row_cur;
    row_cur = row_next;
    row_next = fetch(j + 2);
  }
  // Every copy must land before the CTA may exit. Only the last fill of each slot is still
  // waitable by parity (an earlier one may be two phases back), so each warp waits for its
  // own fills among the last NSLOT of the whole sequence; fills it never issued (after an
  // abort) are skipped.
  const uint32_t all_fills = 2u * n * NP;
  for (uint32_t q = all_fills > (uint32_t)NSLOT ? all_fills - NSLOT : 0; q < issued_end; ++q)
    if ((int)(q % kIssuers) == w)
      drain_wait(full(q % NSLOT), (q / NSLOT) & 1, abort_flag, tmo);
  __syncwarp();
}

// ---------------------------------------------------------------- prefill kernel
template <int D, bool PAGED, bool BF16, bool SQ>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const PrefillArgs a_in, const __grid_constant__ ItemTable items) {
  PrefillArgs a = a_in;  // rebased on one sequence in batched plans and decode
  using C = Cfg<D, SQ>;
  constexpr int NP = C::NP, NSLOT = C::NSLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int64_t qt, kt0, kt1;
  int g, s, slot = kSlotUniform;
  if (a.balanced) {
    const PaItem it = items.item[blockIdx.x];
    const int32_t rb = a.batch > 0 ? batch_rebase<D>(a, items, it.rb) : it.rb;
    rb_coords(rb, a.q_tiles, a.Hkv, &qt, &g);
    s = 0;
    kt0 = it.kt0;
    kt1 = it.kt1;
    slot = it.slot;
  } else if (a.batch > 0) {
    decode_unit<D>(a, reinterpret_cast<int32_t*>(smem + C::RING_OFF), &g, &s, &kt0, &kt1);
    qt = 0;
  } else {
    unit_coords(blockIdx.x, a.q_tiles, a.Hkv, a.splits, &qt, &g, &s);
    split_range(tile_kv_tiles(qt, a.R, a.G, a.hist_len), s, a.splits, &kt0, &kt1);
  }
  const int n = (int)(kt1 - kt0);

  if (n == 0) {  // a split past this tile's keys (only when S > KV tiles): empty partial
    empty_unit<D>(a, qt, g, s);
    return;
  }

  // The copy warps read the page-table entries of the first two KV tiles before the set-up
  // below, so the loads overlap it and the first copies go out right after it.
  int32_t pre_row0 = a.oob_row, pre_row1 = a.oob_row;
  if (warp > kMmaWarp) {
    const bool report = warp == kMmaWarp + 1;
    pre_row0 = tile_page_row<PAGED>(a, kt0, n, 0, lane, report);
    pre_row1 = tile_page_row<PAGED>(a, kt0, n, 1, lane, report);
  }
  auto bar = [&](int i) -> uint32_t { return sb + C::BAR_OFF + 8u * (uint32_t)i; };
  auto slot_addr = [&](uint32_t slot) -> uint32_t { return sb + C::RING_OFF + slot * kPanel; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(bar(C::B_FULL + i), 1);
      mbar_init(bar(C::B_EMPTY + i), 1);
    }
    mbar_init(bar(C::B_QFULL), 4);
    mbar_init(bar(C::B_SFULL + 0), 1);
    mbar_init(bar(C::B_SFULL + 1), 1);
    mbar_init(bar(C::B_PFULL + 0), 4);
    mbar_init(bar(C::B_PFULL + 1), 4);
    mbar_init(bar(C::B_PVDONE + 0), 1);
    mbar_init(bar(C::B_PVDONE + 1), 1);
    mbar_init(bar(C::B_MMADONE), 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp + 1 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;

  if (warp < 4) {
    // ============================================================ softmax + epilogue
    SoftmaxCtx sc;
    sc.sb = sb;
    sc.q_off = C::Q_OFF;
    sc.bar_sfull = bar(C::B_SFULL);
    sc.bar_pvdone = bar(C::B_PVDONE);
    sc.arrive_qfull = bar(C::B_QFULL);
    sc.arrive_pfull = bar(C::B_PFULL);
    sc.remote_arrive = false;
    sc.tmem = tmem;
    sc.qt = qt;
    sc.g = g;
    sc.s = s;
    sc.kt0 = kt0;
    sc.n = n;
    sc.slot = slot;
    sc.row0 = 0;
    sc.stage_off = C::RING_OFF;
    static_assert(C::NSLOT * kPanel >= kTileRows * (D * 4 + 16), "staging needs the ring");
    sc.abort_flag = abort_flag;
    sc.tmo = tmo;
    // Keys past the sequence in its last page hold arbitrary bits; P is 0 there but 0 * NaN
    // is NaN inside the MMA, so those V rows are zeroed before PV reads them.
    auto v_tail = [&](int j, int r) -> bool {
      const uint32_t seq0 = v_item(j, n) * NP;
      bool okv = true;
      for (int p = 0; p < NP && okv; ++p)
        okv = warp_wait(bar(C::B_FULL + (seq0 + p) % NSLOT), ((seq0 + p) / NSLOT) & 1, abort_flag,
                        tmo);
      if (!okv || r < 0) return okv;
      for (int p = 0; p < NP; ++p) {
        const uint32_t off = v_offset<NP, C::PANEL_LOG>((uint32_t)r, p, a.v_shift);
        const uint32_t ra = slot_addr((seq0 + (off >> 14)) % NSLOT) + (off & (kPanel - 1));
#pragma unroll
        for (int c = 0; c < 8; ++c) st_shared_v4(ra + c * 16, 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      return true;
    };
    softmax_role<D, PAGED, BF16, SQ>(a, sc, v_tail);
  } else if (warp > kMmaWarp) {
    // ============================================================ TMA issuers (three warps)
    kv_copy_role<NP, NSLOT, C::PANEL_LOG, PAGED>(a, &tm_k, &tm_v, g, kt0, n,
                                                 warp - kMmaWarp - 1, sb + C::RING_OFF,
                                                 bar(C::B_FULL), bar(C::B_EMPTY), pre_row0,
                                                 pre_row1, abort_flag, tmo);
  } else {
    // ============================================================ MMA issuer (one lane)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_f16(128, kTileKeys, BF16, false);
      constexpr uint32_t idesc_pv = umma_idesc_f16(128, D, BF16, true);
      constexpr uint32_t kSlotDesc = kPanel >> 4;  // descriptor units per slot
      // Descriptor templates; the start address field takes plain additions of (bytes >> 4).
      const uint64_t q_desc = smem_desc_sw128(sb + C::Q_OFF, 16, C::Q_SBO);
      const uint64_t k_desc = smem_desc_sw128(sb + C::RING_OFF, 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(sb + C::RING_OFF, (uint32_t)a.v_rows * 128u, 1024);
      uint32_t slot = 0, round = 0;
      bool ok = thread_wait(bar(C::B_QFULL), 0, abort_flag, tmo);
      tc_fence_after();
      for (int j = 0; j <= n && ok; ++j) {
        if (j < n) {
          // S_j is written over S_{j-2} and its P: the PV MMA that read that P was issued
          // earlier by this thread, and tcgen05.mma executes in issue order.
          const uint32_t s_tmem = tmem + kSCol0 + 128u * (j & 1);
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            ok = thread_wait(bar(C::B_FULL + slot), round & 1, abort_flag, tmo);
            if (!ok) break;
            tc_fence_after();
            const uint64_t ad = q_desc + p * (C::Q_PANEL >> 4), bd = k_desc + slot * kSlotDesc;
            umma_ss(s_tmem, ad, bd, idesc_qk, p != 0 ? 1u : 0u);
            umma_ss(s_tmem, ad + 2, bd + 2, idesc_qk, 1u);
            umma_ss(s_tmem, ad + 4, bd + 4, idesc_qk, 1u);
            umma_ss(s_tmem, ad + 6, bd + 6, idesc_qk, 1u);
            umma_commit(bar(C::B_EMPTY + slot));
            if (++slot == (uint32_t)NSLOT) {
              slot = 0;
              ++round;
            }
          }
          if (!ok) break;
          umma_commit(bar(C::B_SFULL + (j & 1)));
        }
        if (j >= 1) {
          const int i = j - 1;
          ok = thread_wait(bar(C::B_PFULL + (i & 1)), (i >> 1) & 1, abort_flag, tmo);
          const uint32_t vslot0 = slot;  // the V tile takes slots vslot0, vslot0 + 1, ... (mod NSLOT)
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            if (ok) ok = thread_wait(bar(C::B_FULL + slot), round & 1, abort_flag, tmo);
            if (++slot == (uint32_t)NSLOT) {
              slot = 0;
              ++round;
            }
          }
          if (!ok) break;
          tc_fence_after();
          const uint32_t p_tmem = tmem + kSCol0 + 128u * (i & 1) + kPColOff;
#pragma unroll
          for (int ks = 0; ks < kTileKeys / 16; ++ks) {
            const uint32_t off = v_offset<NP, C::PANEL_LOG>(16u * ks, 0, a.v_shift);
            uint32_t vs = vslot0 + (off >> 14);
            if (vs >= (uint32_t)NSLOT) vs -= NSLOT;
            umma_ts(tmem + kOCol, p_tmem + ks * 8,
                    v_desc + vs * kSlotDesc + ((off & (kPanel - 1)) >> 4), idesc_pv,
                    (i > 0 || ks > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < NP; ++k) {
            uint32_t vs = vslot0 + k;
            if (vs >= (uint32_t)NSLOT) vs -= NSLOT;
            umma_commit(bar(C::B_EMPTY + vs));
          }
          umma_commit(bar(C::B_PVDONE + (i & 1)));
        }
      }
      // Every issued MMA must finish before tensor memory is freed.
      umma_commit(bar(C::B_MMADONE));
      drain_wait(bar(C::B_MMADONE), 0, abort_flag, tmo);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

#include "prefill_pair.cuh"
#include "decode_kernel.cuh"
#include "kv_append.cuh"

// ---------------------------------------------------------------- combine kernels
// The merge of one output row (one warp): part p's partial row is at o + p * o_stride (D fp32,
// already divided by its own sum) and its base-2 LSE at lse + p * lse_stride, p < np <= 32.
// Lane p holds LSE p; shuffles give M = max and W = sum of 2^(lse_p - M); the row is
// sum_p 2^(lse_p - M) O_p / W, parts of weight 0 skipped, multiply-adds in part order. Loads
// go out four parts at a time, both 128-column passes together, and the first four are issued
// before the weights are known: one memory latency per four parts, not one per part and pass.
// Every lane takes part in every shuffle (at D = 64 only lanes 0-15 own columns, but the
// weights of parts 16-31 sit in lanes 16-31).
template <int NPASS>  // 128-column passes: 1 for D = 64 and 128, 2 for D = 256
__device__ __forceinline__ void merge_row(const float* __restrict__ o, int64_t o_stride,
                                          const float* __restrict__ lse_p, int64_t lse_stride,
                                          int np, int D, float* __restrict__ dst, int lane) {
  constexpr int kGroup = 4;
  const float lse = lane < np ? lse_p[(int64_t)lane * lse_stride] : -INFINITY;
  float4 v[kGroup][NPASS];
  auto load_group = [&](int p0) {
#pragma unroll
    for (int k = 0; k < kGroup; ++k)
#pragma unroll
      for (int ps = 0; ps < NPASS; ++ps) {
        const int d0 = lane * 4 + 128 * ps;
        v[k][ps] = (p0 + k < np && d0 < D)
                       ? *reinterpret_cast<const float4*>(o + (int64_t)(p0 + k) * o_stride + d0)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
  };
  load_group(0);
  float M = lse;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float wt = (lse == -INFINITY) ? 0.f : exp2f(lse - M);
  float W = wt;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
  const float inv = W > 0.f ? 1.f / W : 0.f;
  float4 acc[NPASS];
#pragma unroll
  for (int ps = 0; ps < NPASS; ++ps) acc[ps] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int p0 = 0; p0 < np; p0 += kGroup) {  // np is the same in every lane
    if (p0 > 0) load_group(p0);
#pragma unroll
    for (int k = 0; k < kGroup; ++k) {
      const float w = __shfl_sync(0xffffffffu, wt, (p0 + k) & 31);
      if (p0 + k < np && w != 0.f) {
#pragma unroll
        for (int ps = 0; ps < NPASS; ++ps) {
          acc[ps].x = fmaf(w, v[k][ps].x, acc[ps].x);
          acc[ps].y = fmaf(w, v[k][ps].y, acc[ps].y);
          acc[ps].z = fmaf(w, v[k][ps].z, acc[ps].z);
          acc[ps].w = fmaf(w, v[k][ps].w, acc[ps].w);
        }
      }
    }
  }
#pragma unroll
  for (int ps = 0; ps < NPASS; ++ps) {
    const int d0 = lane * 4 + 128 * ps;
    if (d0 < D)
      *reinterpret_cast<float4*>(dst + d0) = make_float4(acc[ps].x * inv, acc[ps].y * inv,
                                                         acc[ps].z * inv, acc[ps].w * inv);
  }
}

// Uniform splits: one warp per (row, head) merges its S <= 32 split partials into out.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ ws_o,
                                                      const float* __restrict__ ws_lse,
                                                      float* __restrict__ out, int S, int64_t RH,
                                                      int D) {
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (w >= RH) return;
  const int lane = threadIdx.x & 31;
  if (D == 256)
    merge_row<2>(ws_o + w * D, RH * D, ws_lse + w, RH, S, D, out + w * D, lane);
  else
    merge_row<1>(ws_o + w * D, RH * D, ws_lse + w, RH, S, D, out + w * D, lane);
}

// Balanced plans: one warp per packed row of a cut row block merges that row's parts (workspace
// slots first_slot .. first_slot + nparts - 1, at most 32) into out, with the same weighting.
// Batched plans: the sequences (n_seq > 0), whose row blocks the split blocks name.
struct SplitTable {
  PaSplitBlock blk[kMaxSplitBlocks];
  PaSeq seq[kMaxSeqs];
};

__global__ void __launch_bounds__(256) combine_blocks_kernel(
    const float* __restrict__ ws_o, const float* __restrict__ ws_lse, float* __restrict__ out,
    const __grid_constant__ SplitTable t, int n_blocks, int rows_per_block, int64_t q_units,
    int Hkv, int G, int R, int Hq, int D, int n_seq) {
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (w >= (int64_t)n_blocks * rows_per_block) return;
  const int lane = threadIdx.x & 31;
  const PaSplitBlock b = t.blk[w / rows_per_block];
  const int lr = (int)(w % rows_per_block);
  int32_t rb = b.rb;
  if (n_seq > 0) {  // the owning sequence: its rows, its Q-tile units, its output rows
    const PaSeq sq = t.seq[seq_of_rb(t.seq, n_seq, rb)];
    rb -= sq.rb0;
    R = sq.rows;
    q_units = ceil_div64(q_tiles_for(sq.rows, G), rows_per_block / kTileRows);
    out += (int64_t)sq.q_row0 * Hq * D;
  }
  int64_t qu;
  int g;
  rb_coords(rb, q_units, Hkv, &qu, &g);
  const int64_t grow = qu * rows_per_block + lr;
  const int64_t tok = grow / G;
  if (tok >= R) return;
  const int head = g * G + (int)(grow % G);
  const int64_t row0 = (int64_t)b.first_slot * rows_per_block + lr;  // part p: row0 + p * rpb
  float* dst = out + (tok * Hq + head) * (int64_t)D;
  const int64_t rpb = rows_per_block;
  if (D == 256)
    merge_row<2>(ws_o + row0 * D, rpb * D, ws_lse + row0, rpb, b.nparts, D, dst, lane);
  else
    merge_row<1>(ws_o + row0 * D, rpb * D, ws_lse + row0, rpb, b.nparts, D, dst, lane);
}

// ---------------------------------------------------------------- timeout self-test
__global__ void selftest_timeout_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t never;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&never), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  // Nothing arrives on `never`: the wait gives up after timeout_ns and sets the timeout bit.
  warp_wait(smem_u32(&never), 0, &abort_flag, timeout_ns);
}

// ---------------------------------------------------------------- host side
std::atomic<uint64_t> g_timeout_ns{2000000000ull};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// K as a 3-D tensor {D, Hkv, rows}: a box is 64 elements (128 B, one swizzle row) of one KV
// head for `box_rows` consecutive key rows.
bool make_k_map(CUtensorMap* map, const void* base, bool bf16, int D, int Hkv, int64_t rows,
                int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r =
      fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// V as a 4-D tensor {64, rows, D/64 panels, Hkv}: a box is `panels` 64-wide panels of one KV
// head for `box_rows` key rows, laid out panel after panel in shared memory (each panel a
// column of 128-byte swizzled rows), which is the MN-major operand layout of P V.
bool make_v_map(CUtensorMap* map, const void* base, bool bf16, int D, int Hkv, int64_t rows,
                int box_rows, int panels) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)(D / 64), (cuuint64_t)Hkv};
  const cuuint64_t strides[3] = {(cuuint64_t)Hkv * D * 2, 128, (cuuint64_t)D * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)box_rows, (cuuint32_t)panels, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r =
      fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Q of one piece as a 4-D tensor {D, G, Hkv, R}: a box is 64 elements (one swizzle row) of
// all G heads of KV head g for 128/G tokens, i.e. one panel of a packed 128-row Q tile when
// G divides 128. Rows past the piece read as zeros.
bool make_q_map(CUtensorMap* map, const void* base, bool bf16, int D, int G, int Hkv, int R) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)G, (cuuint64_t)Hkv, (cuuint64_t)R};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)G * D * 2,
                                 (cuuint64_t)Hkv * G * D * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)G, 1, (cuuint32_t)(kTileRows / G)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r =
      fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool PAGED, bool BF16, bool SQ = false>
cudaError_t launch_prefill(int64_t grid, cudaStream_t st, const CUtensorMap& tk,
                           const CUtensorMap& tv, const PrefillArgs& a, const ItemTable& it) {
  auto kern = prefill_kernel<D, PAGED, BF16, SQ>;
  static std::atomic<uint64_t> configured{0};  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<D, SQ>::LAUNCH_SMEM);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  kern<<<(unsigned)grid, kThreads, Cfg<D, SQ>::LAUNCH_SMEM, st>>>(tk, tv, a, it);
  return cudaGetLastError();
}

template <bool PAGED, bool BF16>
cudaError_t launch_pair(int64_t grid, cudaStream_t st, const CUtensorMap& tk,
                        const CUtensorMap& tv, const CUtensorMap& tq, const PrefillArgs& a,
                        const ItemTable& it) {
  auto kern = prefill_pair_kernel<PAGED, BF16>;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairCfg::LAUNCH_SMEM);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = PairCfg::LAUNCH_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, a, it);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(bool paged, bool bf16, int64_t grid, cudaStream_t st, const CUtensorMap& tk,
                     const CUtensorMap& tv, const PrefillArgs& a, const ItemTable& it) {
  if (paged)
    return bf16 ? launch_prefill<D, true, true>(grid, st, tk, tv, a, it)
                : launch_prefill<D, true, false>(grid, st, tk, tv, a, it);
  return bf16 ? launch_prefill<D, false, true>(grid, st, tk, tv, a, it)
              : launch_prefill<D, false, false>(grid, st, tk, tv, a, it);
}

// The decode kernels' attributes (shared memory, carveout for two CTAs per SM), once per device.
template <class K>
cudaError_t configure_decode(K kern, int smem, std::atomic<uint64_t>& configured) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  return cudaSuccess;
}

template <int D, bool BF16, bool BAL>
cudaError_t launch_decode(int64_t grid, cudaStream_t st, const CUtensorMap& tk,
                          const CUtensorMap& tv, const PrefillArgs& a, const ItemTable& it) {
  static std::atomic<uint64_t> configured{0};  // one bit per device ordinal
  cudaError_t e;
  if constexpr (BAL) {
    e = configure_decode(decode_batch_kernel<D, BF16>, DecCfg<D>::LAUNCH_SMEM, configured);
    if (e != cudaSuccess) return e;
    decode_batch_kernel<D, BF16><<<(unsigned)grid, kThreads, DecCfg<D>::LAUNCH_SMEM, st>>>(
        tk, tv, a, it);
  } else {
    e = configure_decode(decode_kernel<D, BF16>, DecCfg<D>::LAUNCH_SMEM, configured);
    if (e != cudaSuccess) return e;
    decode_kernel<D, BF16><<<(unsigned)grid, kThreads, DecCfg<D>::LAUNCH_SMEM, st>>>(tk, tv, a);
  }
  return cudaGetLastError();
}

template <bool BAL>
cudaError_t launch_decode_d(int D, bool bf16, int64_t grid, cudaStream_t st,
                            const CUtensorMap& tk, const CUtensorMap& tv, const PrefillArgs& a,
                            const ItemTable& it) {
  return D == 128 ? (bf16 ? launch_decode<128, true, BAL>(grid, st, tk, tv, a, it)
                          : launch_decode<128, false, BAL>(grid, st, tk, tv, a, it))
                  : (bf16 ? launch_decode<256, true, BAL>(grid, st, tk, tv, a, it)
                          : launch_decode<256, false, BAL>(grid, st, tk, tv, a, it));
}

// Paged single-CTA launches of decode and batches (sq: every Q tile holds <= 8 packed rows).
cudaError_t launch_paged_single(int D, bool bf16, bool sq, int64_t grid, cudaStream_t st,
                                const CUtensorMap& tk, const CUtensorMap& tv,
                                const PrefillArgs& a, const ItemTable& it) {
  if (sq) {
    switch (D) {
      case 64: return bf16 ? launch_prefill<64, true, true, true>(grid, st, tk, tv, a, it)
                           : launch_prefill<64, true, false, true>(grid, st, tk, tv, a, it);
      case 128: return bf16 ? launch_prefill<128, true, true, true>(grid, st, tk, tv, a, it)
                            : launch_prefill<128, true, false, true>(grid, st, tk, tv, a, it);
      default: return bf16 ? launch_prefill<256, true, true, true>(grid, st, tk, tv, a, it)
                           : launch_prefill<256, true, false, true>(grid, st, tk, tv, a, it);
    }
  }
  switch (D) {
    case 64: return launch_d<64>(true, bf16, grid, st, tk, tv, a, it);
    case 128: return launch_d<128>(true, bf16, grid, st, tk, tv, a, it);
    default: return bf16 ? launch_prefill<256, true, true>(grid, st, tk, tv, a, it)
                         : launch_prefill<256, true, false>(grid, st, tk, tv, a, it);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace pa

using namespace pa;

extern "C" int pa_prefill(const pa_plan_t* plan, const void* q, const void* k_pool,
                          const void* v_pool, const int32_t* page_table, int64_t num_pages,
                          int64_t hist_len, int chunk_rows, float* out, float* lse_ws,
                          uint64_t ws_bytes, pa_stream_t stream) {
  if (!plan || !q || !k_pool || !v_pool || plan->batch != 0) return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool)) return PA_ERR_INVALID_ARG;
  if (hist_len != plan->hist_len || chunk_rows != plan->chunk_rows || chunk_rows <= 0)
    return PA_ERR_INVALID_ARG;
  const int D = plan->head_dim;
  if (D != 64 && D != 128 && D != 256) return PA_ERR_UNSUPPORTED;
  if (plan->splits < 1 || plan->splits > PA_MAX_SPLITS || plan->n_kv_heads <= 0 ||
      plan->n_q_heads != plan->n_kv_heads * plan->group)
    return PA_ERR_INVALID_ARG;
  const int64_t total_keys = hist_len + chunk_rows;
  const int S = plan->splits;
  const bool balanced = plan->policy == PA_POLICY_BALANCED;
  Schedule sch;
  if (balanced && (!build_balanced(*plan, &sch) || (int64_t)sch.items.size() != plan->units))
    return PA_ERR_INVALID_ARG;
  const bool partials = balanced ? sch.n_slots > 0 : S > 1;
  if (balanced || S == 1) {
    if (!out || !aligned16(out)) return PA_ERR_INVALID_ARG;
  }
  if (partials) {
    if (!lse_ws || !aligned16(lse_ws) || ws_bytes < plan->ws_bytes) return PA_ERR_WORKSPACE;
  }
  const bool paged = plan->paged != 0;
  const bool bf16 = plan->dtype == PA_BF16;
  const int PS = plan->page_size;
  if (paged) {
    if (!page_table || num_pages <= 0) return PA_ERR_INVALID_ARG;
    if (num_pages * PS + kTileKeys >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  }
  const int per = plan->ctas_per_unit;
  if (per != (D == 256 ? 2 : 1)) return PA_ERR_INVALID_ARG;
  const int64_t q_units = ((int64_t)plan->q_tiles + per - 1) / per;
  const int64_t grid = plan->units * per;  // CTAs
  const int64_t want_units = balanced ? (int64_t)sch.items.size() : q_units * plan->n_kv_heads * S;
  if (plan->units != want_units || grid <= 0 || grid >= (int64_t(1) << 31))
    return PA_ERR_INVALID_ARG;

  CUtensorMap tk, tv;
  const int64_t rows = paged ? num_pages * PS : total_keys;
  const int page_rows = paged ? PS : kTileKeys;  // key rows of one page
  // Single CTA: a K box is a page (one 64-wide panel), a V box covers all of D (<= 16 KB).
  // CTA pair: each CTA loads 64 keys of K and half of D of V, in boxes of <= 64 keys.
  const int k_rows = per == 2 ? std::min(page_rows, 64) : page_rows;
  const int v_rows = per == 2 ? std::min(page_rows, 64) : std::min(page_rows, 128 / (D / 64));
  const int v_panels = per == 2 ? 2 : D / 64;
  // CTA pair, pages of 16 keys: K in boxes of 8 keys x all of D (one swizzle atom per panel),
  // 8 boxes per half tile instead of 16 one-panel boxes of a page each
  const bool k_atoms = per == 2 && page_rows == 16;
  if (!(k_atoms ? make_v_map(&tk, k_pool, bf16, D, plan->n_kv_heads, rows, 8, D / 64)
                : make_k_map(&tk, k_pool, bf16, D, plan->n_kv_heads, rows, k_rows)) ||
      !make_v_map(&tv, v_pool, bf16, D, plan->n_kv_heads, rows, v_rows, v_panels))
    return PA_ERR_CUDA;
  // CTA pair: Q by tensor copy when a packed 128-row tile is whole tokens
  CUtensorMap tq;
  const bool q_tma = per == 2 && kTileRows % plan->group == 0;
  if (q_tma && !make_q_map(&tq, q, bf16, D, plan->group, plan->n_kv_heads, chunk_rows))
    return PA_ERR_CUDA;
  if (!q_tma) memset(&tq, 0, sizeof tq);

  PrefillArgs a;
  memset(&a, 0, sizeof a);
  a.q = static_cast<const uint16_t*>(q);
  a.page_table = page_table;
  a.out = out;
  a.ws_o = partials ? lse_ws : nullptr;
  a.ws_lse = !partials ? nullptr
             : balanced ? lse_ws + (int64_t)sch.n_slots * sch.rows_per_block * D
                        : lse_ws + (int64_t)S * chunk_rows * plan->n_q_heads * D;
  a.hist_len = hist_len;
  a.table_len = paged ? (total_keys + PS - 1) / PS : 0;
  a.total_keys = total_keys;
  a.R = chunk_rows;
  a.Hq = plan->n_q_heads;
  a.Hkv = plan->n_kv_heads;
  a.G = plan->group;
  a.q_tiles = plan->q_tiles;
  a.splits = S;
  a.page_rows = page_rows;
  a.page_shift = __builtin_ctz((unsigned)page_rows);
  a.pages_per_tile = kTileKeys / page_rows;
  a.k_rows = k_rows;
  a.v_rows = v_rows;
  a.v_shift = __builtin_ctz((unsigned)v_rows);
  a.num_pages = paged ? (int32_t)num_pages : 0;
  a.oob_row = (int32_t)rows;
  a.scale_log2 = plan->scale * 1.4426950408889634f;
  a.timeout_ns = g_timeout_ns.load();
  a.balanced = balanced ? 1 : 0;
  a.ws_split_rows = (int64_t)chunk_rows * plan->n_q_heads;
  a.batch = 0;
  a.table_stride = 0;
  a.seq_lens = nullptr;
  a.q_tma = q_tma ? 1 : 0;
  a.k_atoms = k_atoms ? 1 : 0;
  a.rows_per_block = per * kTileRows;
  // Kernel parameter of 8 KB, copied into the launch: kept off the stack of callers with small
  // stacks, one per thread (the launch has taken its copy when this function returns).
  thread_local ItemTable table;
  ItemTable* tab = &table;
  for (size_t i = 0; i < sch.items.size(); ++i) tab->item[i] = sch.items[i];

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (D) {
    case 64: e = launch_d<64>(paged, bf16, grid, st, tk, tv, a, *tab); break;
    case 128: e = launch_d<128>(paged, bf16, grid, st, tk, tv, a, *tab); break;
    default:
      e = paged ? (bf16 ? launch_pair<true, true>(grid, st, tk, tv, tq, a, *tab)
                        : launch_pair<true, false>(grid, st, tk, tv, tq, a, *tab))
                : (bf16 ? launch_pair<false, true>(grid, st, tk, tv, tq, a, *tab)
                        : launch_pair<false, false>(grid, st, tk, tv, tq, a, *tab));
      break;
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_decode(const pa_plan_t* plan, const void* q, const void* k_pool,
                         const void* v_pool, const int32_t* block_table, int table_stride,
                         const int32_t* seq_lens, int64_t num_pages, float* out, float* lse_ws,
                         uint64_t ws_bytes, pa_stream_t stream) {
  if (!plan || plan->batch <= 0 || plan->chunk_rows != plan->batch || plan->q_tiles != 1 ||
      plan->policy == PA_POLICY_BALANCED)  // batch plans run through pa_batch_prefill
    return PA_ERR_INVALID_ARG;
  if (!q || !k_pool || !v_pool || !block_table || !seq_lens || !out || table_stride <= 0 ||
      num_pages <= 0)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  const int D = plan->head_dim, S = plan->splits, B = plan->batch, PS = plan->page_size;
  if (D != 64 && D != 128 && D != 256) return PA_ERR_UNSUPPORTED;
  if (S < 1 || S > PA_MAX_SPLITS || plan->n_q_heads != plan->n_kv_heads * plan->group ||
      plan->group > kTileRows || plan->units != (int64_t)B * plan->n_kv_heads * S)
    return PA_ERR_INVALID_ARG;
  if (S > 1 && (!lse_ws || !aligned16(lse_ws) || ws_bytes < plan->ws_bytes))
    return PA_ERR_WORKSPACE;
  if (num_pages * PS + kTileKeys >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  const bool bf16 = plan->dtype == PA_BF16;
  const int64_t rows = num_pages * PS;
  const int v_rows = std::min(PS, 128 / (D / 64));
  CUtensorMap tk, tv;
  if (!make_k_map(&tk, k_pool, bf16, D, plan->n_kv_heads, rows, PS) ||
      !make_v_map(&tv, v_pool, bf16, D, plan->n_kv_heads, rows, v_rows, D / 64))
    return PA_ERR_CUDA;
  PrefillArgs a;
  memset(&a, 0, sizeof a);
  a.q = static_cast<const uint16_t*>(q);
  a.page_table = block_table;
  a.out = out;
  a.ws_o = S > 1 ? lse_ws : nullptr;
  a.ws_lse = S > 1 ? lse_ws + (int64_t)S * B * plan->n_q_heads * D : nullptr;
  a.R = 1;
  a.Hq = plan->n_q_heads;
  a.Hkv = plan->n_kv_heads;
  a.G = plan->group;
  a.q_tiles = 1;
  a.splits = S;
  a.page_rows = PS;
  a.page_shift = __builtin_ctz((unsigned)PS);
  a.pages_per_tile = kTileKeys / PS;
  a.k_rows = PS;
  a.v_rows = v_rows;
  a.v_shift = __builtin_ctz((unsigned)v_rows);
  a.num_pages = (int32_t)num_pages;
  a.oob_row = (int32_t)rows;
  a.scale_log2 = plan->scale * 1.4426950408889634f;
  a.timeout_ns = g_timeout_ns.load();
  a.rows_per_block = kTileRows;
  a.ws_split_rows = (int64_t)B * plan->n_q_heads;
  a.batch = B;
  a.table_stride = table_stride;
  a.seq_lens = seq_lens;
  thread_local ItemTable table;  // unused by decode units
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t grid = plan->units;
  if (grid >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  cudaError_t e;
  if (decode_swapped(D, plan->group))
    e = launch_decode_d<false>(D, bf16, grid, st, tk, tv, a, table);
  else
    e = launch_paged_single(D, bf16, plan->group <= 8, grid, st, tk, tv, a, table);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_combine(const pa_plan_t* plan, const float* lse_ws, uint64_t ws_bytes,
                          float* out, pa_stream_t stream) {
  if (!plan || (plan->policy == PA_POLICY_BALANCED && plan->batch != 0))
    return PA_ERR_INVALID_ARG;  // batched plans merge with pa_batch_combine
  const int S = plan->splits;
  if (plan->policy == PA_POLICY_BALANCED) {
    Schedule sch;
    if (!build_balanced(*plan, &sch) || (int64_t)sch.items.size() != plan->units)
      return PA_ERR_INVALID_ARG;
    if (sch.split.empty()) return PA_OK;
    if (sch.max_parts > 32) return PA_ERR_INVALID_ARG;
    if (!lse_ws || ws_bytes < plan->ws_bytes || !aligned16(lse_ws)) return PA_ERR_WORKSPACE;
    if (!out || !aligned16(out)) return PA_ERR_INVALID_ARG;
    thread_local SplitTable table;
    for (size_t i = 0; i < sch.split.size(); ++i) table.blk[i] = sch.split[i];
    const int D = plan->head_dim;
    const int per = plan->ctas_per_unit;
    const int64_t q_units = ((int64_t)plan->q_tiles + per - 1) / per;
    const int64_t warps = (int64_t)sch.split.size() * sch.rows_per_block;
    combine_blocks_kernel<<<(unsigned)((warps + 7) / 8), 256, 0,
                            reinterpret_cast<cudaStream_t>(stream)>>>(
        lse_ws, lse_ws + (int64_t)sch.n_slots * sch.rows_per_block * D, out, table,
        (int)sch.split.size(), sch.rows_per_block, q_units, plan->n_kv_heads, plan->group,
        plan->chunk_rows, plan->n_q_heads, D, 0);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  if (S == 1) return PA_OK;
  if (S < 1 || S > PA_MAX_SPLITS) return PA_ERR_INVALID_ARG;
  if (!lse_ws || ws_bytes < plan->ws_bytes || !aligned16(lse_ws)) return PA_ERR_WORKSPACE;
  if (!out || !aligned16(out)) return PA_ERR_INVALID_ARG;
  const int D = plan->head_dim;
  const int64_t RH = (int64_t)plan->chunk_rows * plan->n_q_heads;
  const float* ws_o = lse_ws;
  const float* ws_lse = lse_ws + (int64_t)S * RH * D;
  const int64_t blocks = (RH + 7) / 8;
  combine_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      ws_o, ws_lse, out, S, RH, D);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------- batched prefill
namespace pa {
// The batch and its schedule, rebuilt from the caller's lengths and checked against the plan.
static int rebuild_batch(const pa_plan_t* plan, const int32_t* q_lens, const int64_t* hist_lens,
                         Batch* bt, Schedule* sch) {
  if (!plan || plan->batch <= 0 || plan->policy != PA_POLICY_BALANCED || !q_lens || !hist_lens)
    return PA_ERR_INVALID_ARG;
  if (plan->batch > kMaxSeqs) return PA_ERR_UNSUPPORTED;
  const int D = plan->head_dim;
  if (D != 64 && D != 128 && D != 256) return PA_ERR_UNSUPPORTED;
  if (plan->n_kv_heads <= 0 || plan->n_q_heads != plan->n_kv_heads * plan->group ||
      plan->ctas_per_unit != batch_ctas_per_unit(D, plan->group, plan->batch, q_lens))
    return PA_ERR_INVALID_ARG;
  const int st = describe_batch(plan->batch, q_lens, hist_lens, plan->group, plan->n_kv_heads,
                                plan->ctas_per_unit, bt);
  if (st != PA_OK) return st;
  if (!build_batch(plan->num_sms, D, plan->ctas_per_unit, plan->group, plan->n_kv_heads, *bt,
                   sch) ||
      (int64_t)sch->items.size() != plan->units || bt->total_rows != plan->chunk_rows ||
      (uint64_t)sch->n_slots * sch->rows_per_block * (D + 1) * 4ull != plan->ws_bytes)
    return PA_ERR_INVALID_ARG;
  return PA_OK;
}
}  // namespace pa

extern "C" int pa_batch_prefill(const pa_plan_t* plan, const int32_t* q_lens,
                                const int64_t* hist_lens, const void* q, const void* k_pool,
                                const void* v_pool, const int32_t* block_table, int table_stride,
                                int64_t num_pages, float* out, float* lse_ws, uint64_t ws_bytes,
                                pa_stream_t stream) {
  Batch bt;
  Schedule sch;
  const int st = rebuild_batch(plan, q_lens, hist_lens, &bt, &sch);
  if (st != PA_OK) return st;
  if (!q || !k_pool || !v_pool || !block_table || !out || table_stride <= 0 || num_pages <= 0)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out))
    return PA_ERR_INVALID_ARG;
  for (const PaSeq& sq : bt.seq)  // every sequence's pages fit its table row
    if (ceil_div64((int64_t)sq.hist + sq.rows, plan->page_size) > table_stride)
      return PA_ERR_INVALID_ARG;
  if (sch.n_slots > 0 && (!lse_ws || !aligned16(lse_ws) || ws_bytes < plan->ws_bytes))
    return PA_ERR_WORKSPACE;
  const int D = plan->head_dim, PS = plan->page_size, per = plan->ctas_per_unit;
  if (num_pages * PS + kTileKeys >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  const bool bf16 = plan->dtype == PA_BF16;
  const int64_t rows = num_pages * PS;
  const int k_rows = per == 2 ? std::min(PS, 64) : PS;
  const int v_rows = per == 2 ? std::min(PS, 64) : std::min(PS, 128 / (D / 64));
  const int v_panels = per == 2 ? 2 : D / 64;
  const bool k_atoms = per == 2 && PS == 16;  // as in pa_prefill
  CUtensorMap tk, tv, tq;
  if (!(k_atoms ? make_v_map(&tk, k_pool, bf16, D, plan->n_kv_heads, rows, 8, D / 64)
                : make_k_map(&tk, k_pool, bf16, D, plan->n_kv_heads, rows, k_rows)) ||
      !make_v_map(&tv, v_pool, bf16, D, plan->n_kv_heads, rows, v_rows, v_panels))
    return PA_ERR_CUDA;
  const bool q_tma = per == 2 && kTileRows % plan->group == 0;
  if (q_tma && !make_q_map(&tq, q, bf16, D, plan->group, plan->n_kv_heads, (int)bt.total_rows))
    return PA_ERR_CUDA;
  if (!q_tma) memset(&tq, 0, sizeof tq);

  PrefillArgs a;
  memset(&a, 0, sizeof a);
  a.q = static_cast<const uint16_t*>(q);
  a.page_table = block_table;
  a.out = out;
  a.ws_o = sch.n_slots > 0 ? lse_ws : nullptr;
  a.ws_lse = sch.n_slots > 0 ? lse_ws + (int64_t)sch.n_slots * sch.rows_per_block * D : nullptr;
  a.Hq = plan->n_q_heads;
  a.Hkv = plan->n_kv_heads;
  a.G = plan->group;
  a.splits = 1;
  a.page_rows = PS;
  a.page_shift = __builtin_ctz((unsigned)PS);
  a.pages_per_tile = kTileKeys / PS;
  a.k_rows = k_rows;
  a.v_rows = v_rows;
  a.v_shift = __builtin_ctz((unsigned)v_rows);
  a.num_pages = (int32_t)num_pages;
  a.oob_row = (int32_t)rows;
  a.scale_log2 = plan->scale * 1.4426950408889634f;
  a.timeout_ns = g_timeout_ns.load();
  a.balanced = 1;
  a.rows_per_block = per * kTileRows;
  a.q_tma = q_tma ? 1 : 0;
  a.k_atoms = k_atoms ? 1 : 0;
  a.batch = plan->batch;
  a.table_stride = table_stride;
  thread_local ItemTable table;
  for (size_t i = 0; i < sch.items.size(); ++i) table.item[i] = sch.items[i];
  for (size_t i = 0; i < bt.seq.size(); ++i) table.seq[i] = bt.seq[i];
  const int64_t grid = plan->units * per;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int max_rows = 0;  // small Q when no sequence's Q tile holds more than 8 packed rows
  for (const PaSeq& sq : bt.seq) max_rows = std::max(max_rows, (int)sq.rows);
  const bool small_q = (int64_t)max_rows * plan->group <= 8;
  cudaError_t e;
  if (per == 2)
    e = bf16 ? launch_pair<true, true>(grid, cs, tk, tv, tq, a, table)
             : launch_pair<true, false>(grid, cs, tk, tv, tq, a, table);
  else if (batch_decode_swapped(D, plan->group, per, bt.seq.data(), (int)bt.seq.size()))
    e = launch_decode_d<true>(D, bf16, grid, cs, tk, tv, a, table);
  else
    e = launch_paged_single(D, bf16, small_q, grid, cs, tk, tv, a, table);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_batch_combine(const pa_plan_t* plan, const int32_t* q_lens,
                                const int64_t* hist_lens, const float* lse_ws, uint64_t ws_bytes,
                                float* out, pa_stream_t stream) {
  Batch bt;
  Schedule sch;
  const int st = rebuild_batch(plan, q_lens, hist_lens, &bt, &sch);
  if (st != PA_OK) return st;
  if (sch.split.empty()) return PA_OK;
  if (!lse_ws || ws_bytes < plan->ws_bytes || !aligned16(lse_ws)) return PA_ERR_WORKSPACE;
  if (!out || !aligned16(out)) return PA_ERR_INVALID_ARG;
  thread_local SplitTable table;
  for (size_t i = 0; i < sch.split.size(); ++i) table.blk[i] = sch.split[i];
  for (size_t i = 0; i < bt.seq.size(); ++i) table.seq[i] = bt.seq[i];
  const int D = plan->head_dim;
  const int64_t warps = (int64_t)sch.split.size() * sch.rows_per_block;
  combine_blocks_kernel<<<(unsigned)((warps + 7) / 8), 256, 0,
                          reinterpret_cast<cudaStream_t>(stream)>>>(
      lse_ws, lse_ws + (int64_t)sch.n_slots * sch.rows_per_block * D, out, table,
      (int)sch.split.size(), sch.rows_per_block, 0, plan->n_kv_heads, plan->group, 0,
      plan->n_q_heads, D, (int)bt.seq.size());
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ---------------------------------------------------------------- entry point without allocation
// Scratch of pa_prefill_noalloc: the split partials and their log-sum-exps live in this
// file-scope device array (every device that loads the library holds it until exit), so the
// entry point needs no allocation at all. Host code may not pass the symbol itself to a
// kernel (on the host it is only a stand-in, not a device address): its device address is
// looked up once per device with cudaGetSymbolAddress, with that device current.
static __device__ __align__(256) float g_noalloc_ws[PA_NOALLOC_WS_BYTES / sizeof(float)];
static std::mutex g_noalloc_mu;
static float* g_noalloc_ptr[64];  // per device ordinal; null until its first call

static int noalloc_scratch(float** ws) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return PA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) return PA_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *ws = g_noalloc_ptr[dev];
  return PA_OK;
}

extern "C" int pa_prefill_noalloc(const pa_plan_t* plan, const void* q, const void* k_pool,
                                  const void* v_pool, const int32_t* page_table, int64_t num_pages,
                                  int64_t hist_len, int chunk_rows, float* out,
                                  pa_stream_t stream) {
  if (!plan) return PA_ERR_INVALID_ARG;
  float* ws = nullptr;
  uint64_t ws_bytes = 0;
  if (plan->ws_bytes > 0) {
    if (plan->ws_bytes > PA_NOALLOC_WS_BYTES) return PA_ERR_WORKSPACE;
    const int st = noalloc_scratch(&ws);
    if (st != PA_OK) return st;
    ws_bytes = PA_NOALLOC_WS_BYTES;
  }
  const int st = pa_prefill(plan, q, k_pool, v_pool, page_table, num_pages, hist_len, chunk_rows,
                            out, ws, ws_bytes, stream);
  if (st != PA_OK) return st;
  return pa_combine(plan, ws, ws_bytes, out, stream);
}

extern "C" int pa_kv_append(int n_kv_heads, int head_dim, int page_size, int dtype,
                            const void* k_new, const void* v_new, void* k_pool, void* v_pool,
                            const int32_t* page_table, int64_t num_pages, int64_t hist_len,
                            int chunk_rows, pa_stream_t stream) {
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID_ARG;
  if (n_kv_heads <= 0 || hist_len < 0 || chunk_rows < 0 || num_pages <= 0)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (page_size < 16 || page_size > 128 || (page_size & (page_size - 1))) return PA_ERR_UNSUPPORTED;
  if (chunk_rows == 0) return PA_OK;
  if (!k_new || !v_new || !k_pool || !v_pool || !page_table) return PA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
    return PA_ERR_INVALID_ARG;
  const int row_vecs = n_kv_heads * head_dim * 2 / 16;
  const int64_t pieces = (int64_t)chunk_rows * row_vecs;  // 16-byte pieces per tensor
  const int64_t warps = (pieces + 32 * kAppendBatch - 1) / (32 * kAppendBatch);
  const int64_t blocks = (warps + 7) / 8;
  if (blocks >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  kv_append_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), page_table, num_pages, hist_len,
      chunk_rows, page_size, row_vecs);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_kv_publish(int n_kv_heads, int head_dim, int page_size, int dtype,
                             const void* k_staged, const void* v_staged, void* k_pool,
                             void* v_pool, const int32_t* page_table, int64_t num_pages,
                             int64_t first_pos, int rows, pa_stream_t stream) {
  if (!k_staged || !v_staged || first_pos < 0) return PA_ERR_INVALID_ARG;
  const int64_t off = first_pos * n_kv_heads * head_dim * 2;  // bytes of the rows before
  return pa_kv_append(n_kv_heads, head_dim, page_size, dtype,
                      static_cast<const uint8_t*>(k_staged) + off,
                      static_cast<const uint8_t*>(v_staged) + off, k_pool, v_pool, page_table,
                      num_pages, first_pos, rows, stream);
}

extern "C" int pa_device_error(int* flags, int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_pa_error_flags, sizeof v) != cudaSuccess) return PA_ERR_CUDA;
  if (reset) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(g_pa_error_flags, &zero, sizeof zero) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  if (flags) *flags = (int)v;
  if (v & kFlagPage) return PA_ERR_PAGE_INDEX;
  if (v & kFlagTimeout) return PA_ERR_TIMEOUT;
  return PA_OK;
}

extern "C" void pa_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns ? ns : 1); }

extern "C" int pa_selftest_timeout(uint64_t timeout_ns, pa_stream_t stream) {
  selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
