// pa_kernels.cu — sm_100a kernels of libpa and their C-ABI entry points.
//
// prefill_kernel: one CTA per (KV head, packed Q tile, history split) unit.
//   The operation is prefill attention of a query chunk against a long history read through
//   a paged KV cache (BaseRT issue #51, "Results"), with the history of a piece cut into
//   splits whose partials a reduce merges (splash PR #33, "What changed"). The B200 design:
//   * warp 4 (producer) reads the page table and issues one TMA box per (page, 64-wide
//     D panel) into a ring of 16 KB, 128-byte-swizzled shared-memory panels;
//   * warp 5 (MMA) issues tcgen05.mma: S = Q K^T into one of two tensor-memory S buffers,
//     then O += P V into a tensor-memory O accumulator (fp32);
//   * warps 0-3 (softmax, one thread per packed Q row = tensor-memory lane) load the GQA-
//     packed Q tile, read S with tcgen05.ld, apply the causal mask by select, keep the
//     running max and sum (rescaling O only when the max grows by more than 2^8), write P
//     (rounded to the input type) to shared memory, and finally write O / l (fp32) or the
//     split partial and its base-2 log-sum-exp.
//   Every wait is bounded: on expiry the kernel sets the timeout bit, abandons its work,
//   waits for its own copies and MMAs in flight, frees tensor memory and exits.
// combine_kernel: one warp per (row, head) merges the S partials with a log-sum-exp
//   weighting (the "reduce" of splash PR #33).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "pa.h"
#include "pa_geometry.h"
#include "sm100.cuh"

namespace pa {

__device__ unsigned int g_pa_error_flags;
constexpr unsigned kFlagPage = 1u;
constexpr unsigned kFlagTimeout = 2u;

constexpr int kPanel = 128 * 128;          // bytes of one 128-row x 128-byte panel
constexpr int kThreads = 192;              // 4 softmax warps, 1 producer warp, 1 MMA warp
constexpr float kRescaleLog2 = 8.0f;       // rescale O only when the max grows by > 2^8
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0;              // O accumulator: columns [0, D)
constexpr uint32_t kSCol0 = 256;           // S buffers: [256, 384) and [384, 512)

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
  int32_t page_size;
  int32_t pages_per_tile;
  int32_t num_pages;
  int32_t oob_row;       // a key-row coordinate past the pool: the TMA fills zeros there
  float scale_log2;      // softmax scale * log2(e)
  uint64_t timeout_ns;
};

template <int D>
struct Cfg {
  static constexpr int NP = D / 64;                 // 64-element panels per K/V/Q row
  static constexpr int NSLOT = (D == 256) ? 8 : 10; // ring of 16 KB panels (multiple of NP)
  static constexpr int Q_OFF = 0;
  static constexpr int P_OFF = Q_OFF + NP * kPanel;
  static constexpr int RING_OFF = P_OFF + 2 * kPanel;
  static constexpr int BAR_OFF = RING_OFF + NSLOT * kPanel;
  // barriers: full[NSLOT], empty[NSLOT], q_full, s_full[2], s_free[2], p_full, pv_done, mma_done
  static constexpr int B_FULL = 0, B_EMPTY = NSLOT, B_QFULL = 2 * NSLOT, B_SFULL = 2 * NSLOT + 1,
                       B_SFREE = 2 * NSLOT + 3, B_PFULL = 2 * NSLOT + 5,
                       B_PVDONE = 2 * NSLOT + 6, B_MMADONE = 2 * NSLOT + 7, N_BARS = 2 * NSLOT + 8;
  static constexpr int MISC_OFF = BAR_OFF + 8 * N_BARS;
  static constexpr int SMEM = MISC_OFF + 16;
  static constexpr int LAUNCH_SMEM = SMEM + 1024;   // slack to align the base to 1024 B
  static_assert(NSLOT % NP == 0, "a V tile's panels must not wrap around the ring");
  static_assert(LAUNCH_SMEM <= 232448, "exceeds 227 KB of shared memory per CTA");
};

// Position of tile j's V panels in the load order K0, K1, V0, K2, V1, ..., V_{n-1}.
__device__ __forceinline__ uint32_t v_item(int j, int n) {
  return j == n - 1 ? 2u * n - 1u : 2u * j + 2u;
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
  __syncwarp();
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack_round(float a, float b, float& sum) {
  if constexpr (BF16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    sum += __low2float(h) + __high2float(h);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __half2 h = __floats2half2_rn(a, b);
    sum += __low2float(h) + __high2float(h);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

// ---------------------------------------------------------------- prefill kernel
template <int D, bool PAGED, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const PrefillArgs a) {
  using C = Cfg<D>;
  constexpr int NP = C::NP, NSLOT = C::NSLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int64_t qt;
  int g, s;
  unit_coords(blockIdx.x, a.q_tiles, a.Hkv, a.splits, &qt, &g, &s);
  const int64_t n_kt_all = tile_kv_tiles(qt, a.R, a.G, a.hist_len);
  int64_t kt0, kt1;
  split_range(n_kt_all, s, a.splits, &kt0, &kt1);
  const int n = (int)(kt1 - kt0);

  if (n == 0) {  // a split past this tile's keys (only when S > KV tiles): empty partial
    if (threadIdx.x < kTileRows) {
      const int64_t grow = qt * kTileRows + threadIdx.x;
      const int64_t tok = grow / a.G;
      if (tok < a.R) {
        const int head = g * a.G + (int)(grow % a.G);
        const int64_t row = ((int64_t)s * a.R + tok) * a.Hq + head;
        float4* d4 = reinterpret_cast<float4*>(a.ws_o + row * D);
        for (int i = 0; i < D / 4; ++i) d4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        a.ws_lse[row] = -INFINITY;
      }
    }
    return;
  }

  auto bar = [&](int i) -> uint32_t { return sb + C::BAR_OFF + 8u * (uint32_t)i; };
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
    mbar_init(bar(C::B_SFREE + 0), 4);
    mbar_init(bar(C::B_SFREE + 1), 4);
    mbar_init(bar(C::B_PFULL), 4);
    mbar_init(bar(C::B_PVDONE), 1);
    mbar_init(bar(C::B_MMADONE), 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 5) {
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
    const int r = threadIdx.x;  // packed Q row = tensor-memory lane
    const int64_t grow = qt * kTileRows + r;
    const int64_t tok = grow / a.G;
    const bool valid = tok < a.R;
    const int head = g * a.G + (int)(grow % a.G);
    {
      // Q tile -> shared memory as K-major rows of 64-element panels, 128-byte swizzle.
      const uint4* src =
          reinterpret_cast<const uint4*>(a.q + (valid ? (tok * a.Hq + head) * (int64_t)D : 0));
#pragma unroll
      for (int p = 0; p < NP; ++p) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = valid ? __ldg(src + p * 8 + c) : make_uint4(0u, 0u, 0u, 0u);
          st_shared_v4(sb + C::Q_OFF + p * kPanel + r * 128 + ((c ^ (r & 7)) << 4), v.x, v.y, v.z,
                       v.w);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_QFULL));
    }

    const int64_t limit = valid ? a.hist_len + tok : -1;  // last key this row may see
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    float m_run = -INFINITY;  // running max of scale*log2(e)*score
    float l_run = 0.f;        // running sum of the rounded probabilities
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sbuf = j & 1;
      const int64_t key0 = (kt0 + j) * kTileKeys;
      if (!warp_wait(bar(C::B_SFULL + sbuf), (j >> 1) & 1, abort_flag, tmo)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kTileKeys];
#pragma unroll
      for (int c = 0; c < kTileKeys / 32; ++c)
        tmem_ld32(t_lane + kSCol0 + 128u * sbuf + 32u * c,
                  *reinterpret_cast<float(*)[32]>(&sv[32 * c]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_SFREE + sbuf));

      // causal mask by select (masked scores become -inf, whatever bits they held)
      const int64_t rel64 = limit - key0;
      if (rel64 < kTileKeys - 1) {
        const int rel = rel64 < -1 ? -1 : (int)rel64;
#pragma unroll
        for (int c = 0; c < kTileKeys; ++c)
          if (c > rel) sv[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTileKeys; ++c) mx = fmaxf(mx, sv[c]);
      const float m_new = fmaxf(m_run, mx * a.scale_log2);
      const bool need = m_new > m_run + kRescaleLog2;
      if (j == 0) {
        if (need) m_run = m_new;
      } else if (__any_sync(0xffffffffu, need)) {
        // O must not change under a running MMA: wait for PV of the previous tile.
        if (!warp_wait(bar(C::B_PVDONE), (j - 1) & 1, abort_flag, tmo)) {
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
      uint32_t pk[kTileKeys / 2];
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < kTileKeys; c += 2) {
        const float p0 = ex2(fmaf(sv[c], a.scale_log2, -m_use));
        const float p1 = ex2(fmaf(sv[c + 1], a.scale_log2, -m_use));
        pk[c / 2] = pack_round<BF16>(p0, p1, lsum);
      }
      l_run += lsum;

      // P is single-buffered: PV of the previous tile must be done reading it.
      if (j >= 1 && !warp_wait(bar(C::B_PVDONE), (j - 1) & 1, abort_flag, tmo)) {
        ok = false;
        break;
      }
      if constexpr (PAGED) {
        // Keys past the sequence in its last page hold arbitrary bits; P is 0 there but
        // 0 * NaN is NaN inside the MMA, so those V rows are zeroed before PV reads them.
        if (key0 + kTileKeys > a.total_keys) {
          const uint32_t seq0 = v_item(j, n) * NP;
          bool okv = true;
          for (int p = 0; p < NP && okv; ++p)
            okv = warp_wait(bar(C::B_FULL + (seq0 + p) % NSLOT), ((seq0 + p) / NSLOT) & 1,
                            abort_flag, tmo);
          if (!okv) {
            ok = false;
            break;
          }
          if (key0 + r >= a.total_keys) {
            for (int p = 0; p < NP; ++p) {
              const uint32_t row_addr =
                  sb + C::RING_OFF + ((seq0 + p) % NSLOT) * kPanel + r * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c) st_shared_v4(row_addr + c * 16, 0u, 0u, 0u, 0u);
            }
          }
        }
      }
      // P row -> shared memory: two 64-key K-major panels, 128-byte swizzle.
#pragma unroll
      for (int c = 0; c < kTileKeys / 8; ++c) {
        const int pp = c >> 3, cc = c & 7;
        st_shared_v4(sb + C::P_OFF + pp * kPanel + r * 128 + ((cc ^ (r & 7)) << 4), pk[4 * c],
                     pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PFULL));
    }

    if (ok) ok = warp_wait(bar(C::B_PVDONE), (n - 1) & 1, abort_flag, tmo);
    if (ok) {
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      float* dst = (a.splits == 1) ? a.out + (tok * a.Hq + head) * (int64_t)D
                                   : a.ws_o + (((int64_t)s * a.R + tok) * a.Hq + head) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(t_lane + kOCol + 32u * c, o);
        tmem_wait_ld();
        if (valid) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] = make_float4(o[4 * i] * inv_l, o[4 * i + 1] * inv_l, o[4 * i + 2] * inv_l,
                                o[4 * i + 3] * inv_l);
        }
      }
      if (valid && a.splits > 1)
        a.ws_lse[((int64_t)s * a.R + tok) * a.Hq + head] =
            l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
    }
  } else if (warp == 4) {
    // ============================================================ TMA producer
    const int ppt = PAGED ? a.pages_per_tile : 1;
    uint32_t seq = 0;
    bool ok = true;
    // Raw page-table entries of this lane's page in tiles j-1, j, j+1 (read one tile ahead).
    auto fetch = [&](int jt) -> int32_t {
      if (!PAGED || jt >= n || lane >= ppt) return -1;
      const int64_t lp = (kt0 + jt) * ppt + lane;
      return lp < a.table_len ? __ldg(a.page_table + lp) : -1;
    };
    auto load_item = [&](const CUtensorMap* map, int jt, int32_t entry) -> bool {
      int32_t row_lane = a.oob_row;
      if constexpr (PAGED) {
        const int64_t lp = (kt0 + jt) * ppt + lane;
        if (lane < ppt && lp < a.table_len) {
          if (entry >= 0 && entry < a.num_pages)
            row_lane = entry * a.page_size;
          else
            atomicOr(&g_pa_error_flags, kFlagPage);
        }
      }
      const int32_t key0 = (int32_t)((kt0 + jt) * kTileKeys);
      for (int p = 0; p < NP; ++p) {
        const uint32_t slot = seq % NSLOT;
        if (seq >= (uint32_t)NSLOT &&
            !warp_wait(bar(C::B_EMPTY + slot), ((seq / NSLOT) - 1) & 1, abort_flag, tmo))
          return false;
        int32_t rows[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) rows[i] = __shfl_sync(0xffffffffu, row_lane, i);
        if (lane == 0) {
          const uint32_t full = bar(C::B_FULL + slot);
          const uint32_t dst = sb + C::RING_OFF + slot * kPanel;
          mbar_arrive_expect_tx(full, kPanel);
          if constexpr (PAGED) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < ppt) tma_load_3d(dst + i * a.page_size * 128, map, full, p * 64, g, rows[i]);
          } else {
            tma_load_3d(dst, map, full, p * 64, g, key0);
          }
        }
        __syncwarp();
        ++seq;
      }
      return true;
    };
    int32_t e_prev = -1, e_cur = fetch(0), e_next = fetch(1);
    for (int j = 0; j <= n && ok; ++j) {
      if (j < n) ok = load_item(&tm_k, j, e_cur);
      if (ok && j >= 1) ok = load_item(&tm_v, j - 1, e_prev);
      e_prev = e_cur;
      e_cur = e_next;
      e_next = fetch(j + 2);
    }
    // Every issued copy must land before the CTA may exit.
    for (uint32_t qn = seq > (uint32_t)NSLOT ? seq - NSLOT : 0; qn < seq; ++qn)
      drain_wait(bar(C::B_FULL + qn % NSLOT), (qn / NSLOT) & 1, abort_flag, tmo);
  } else {
    // ============================================================ MMA issuer
    const uint32_t idesc_qk = umma_idesc_f16(128, kTileKeys, BF16, false);
    const uint32_t idesc_pv = umma_idesc_f16(128, D, BF16, true);
    bool ok = warp_wait(bar(C::B_QFULL), 0, abort_flag, tmo);
    tc_fence_after();
    uint32_t seq = 0;
    for (int j = 0; j <= n && ok; ++j) {
      if (j < n) {
        const int sbuf = j & 1;
        if (j >= 2) {
          ok = warp_wait(bar(C::B_SFREE + sbuf), ((j - 2) >> 1) & 1, abort_flag, tmo);
          if (!ok) break;
          tc_fence_after();
        }
        for (int p = 0; p < NP; ++p) {
          const uint32_t slot = seq % NSLOT;
          ok = warp_wait(bar(C::B_FULL + slot), (seq / NSLOT) & 1, abort_flag, tmo);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ss(tmem + kSCol0 + 128u * sbuf,
                      smem_desc_sw128(sb + C::Q_OFF + p * kPanel + kk * 32, 16, 1024),
                      smem_desc_sw128(sb + C::RING_OFF + slot * kPanel + kk * 32, 16, 1024),
                      idesc_qk, (p | kk) != 0);
            umma_commit(bar(C::B_EMPTY + slot));
          }
          __syncwarp();
          ++seq;
        }
        if (!ok) break;
        if (lane == 0) umma_commit(bar(C::B_SFULL + sbuf));
        __syncwarp();
      }
      if (j >= 1) {
        const int i = j - 1;
        ok = warp_wait(bar(C::B_PFULL), i & 1, abort_flag, tmo);
        for (int p = 0; p < NP && ok; ++p)
          ok = warp_wait(bar(C::B_FULL + (seq + p) % NSLOT), ((seq + p) / NSLOT) & 1, abort_flag,
                         tmo);
        if (!ok) break;
        tc_fence_after();
        const uint32_t slot0 = seq % NSLOT;
        if (lane == 0) {
#pragma unroll
          for (int ks = 0; ks < kTileKeys / 16; ++ks)
            umma_ss(tmem + kOCol,
                    smem_desc_sw128(sb + C::P_OFF + (ks >> 2) * kPanel + (ks & 3) * 32, 16, 1024),
                    smem_desc_sw128(sb + C::RING_OFF + slot0 * kPanel + ks * 2048, kPanel, 1024),
                    idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
          for (int p = 0; p < NP; ++p) umma_commit(bar(C::B_EMPTY + (seq + p) % NSLOT));
          umma_commit(bar(C::B_PVDONE));
        }
        __syncwarp();
        seq += NP;
      }
    }
    // Every issued MMA must finish before tensor memory is freed.
    if (lane == 0) umma_commit(bar(C::B_MMADONE));
    __syncwarp();
    drain_wait(bar(C::B_MMADONE), 0, abort_flag, tmo);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- combine kernel
// One warp per (row, head): lanes hold the S <= 32 split LSEs, the warp reduces max and sum
// by shuffles, then each lane accumulates 4 output columns per step.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ ws_o,
                                                      const float* __restrict__ ws_lse,
                                                      float* __restrict__ out, int S, int64_t RH,
                                                      int D) {
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (w >= RH) return;
  const int lane = threadIdx.x & 31;
  const float lse = lane < S ? ws_lse[(int64_t)lane * RH + w] : -INFINITY;
  float M = lse;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float wt = (lse == -INFINITY) ? 0.f : exp2f(lse - M);
  float W = wt;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
  const float inv = W > 0.f ? 1.f / W : 0.f;
  for (int d0 = lane * 4; d0 < D; d0 += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp = 0; sp < S; ++sp) {
      const float ws = __shfl_sync(0xffffffffu, wt, sp);
      if (ws != 0.f) {
        const float4 o = *reinterpret_cast<const float4*>(ws_o + ((int64_t)sp * RH + w) * D + d0);
        acc.x = fmaf(ws, o.x, acc.x);
        acc.y = fmaf(ws, o.y, acc.y);
        acc.z = fmaf(ws, o.z, acc.z);
        acc.w = fmaf(ws, o.w, acc.w);
      }
    }
    *reinterpret_cast<float4*>(out + w * D + d0) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
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

// K or V as a 3-D tensor {D, Hkv, rows}; a box is 64 elements (128 B, one swizzle row) of
// one KV head for `box_rows` consecutive key rows.
bool make_kv_map(CUtensorMap* map, const void* base, bool bf16, int D, int Hkv, int64_t rows,
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

template <int D, bool PAGED, bool BF16>
cudaError_t launch_prefill(int64_t grid, cudaStream_t st, const CUtensorMap& tk,
                           const CUtensorMap& tv, const PrefillArgs& a) {
  auto kern = prefill_kernel<D, PAGED, BF16>;
  static std::atomic<uint64_t> configured{0};  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<D>::LAUNCH_SMEM);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  kern<<<(unsigned)grid, kThreads, Cfg<D>::LAUNCH_SMEM, st>>>(tk, tv, a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(bool paged, bool bf16, int64_t grid, cudaStream_t st, const CUtensorMap& tk,
                     const CUtensorMap& tv, const PrefillArgs& a) {
  if (paged)
    return bf16 ? launch_prefill<D, true, true>(grid, st, tk, tv, a)
                : launch_prefill<D, true, false>(grid, st, tk, tv, a);
  return bf16 ? launch_prefill<D, false, true>(grid, st, tk, tv, a)
              : launch_prefill<D, false, false>(grid, st, tk, tv, a);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace pa

using namespace pa;

extern "C" int pa_prefill(const pa_plan_t* plan, const void* q, const void* k_pool,
                          const void* v_pool, const int32_t* page_table, int64_t num_pages,
                          int64_t hist_len, int chunk_rows, float* out, float* lse_ws,
                          uint64_t ws_bytes, pa_stream_t stream) {
  if (!plan || !q || !k_pool || !v_pool) return PA_ERR_INVALID_ARG;
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
  if (S == 1) {
    if (!out || !aligned16(out)) return PA_ERR_INVALID_ARG;
  } else {
    if (!lse_ws || !aligned16(lse_ws) || ws_bytes < plan->ws_bytes) return PA_ERR_WORKSPACE;
  }
  const bool paged = plan->paged != 0;
  const bool bf16 = plan->dtype == PA_BF16;
  const int PS = plan->page_size;
  if (paged) {
    if (!page_table || num_pages <= 0) return PA_ERR_INVALID_ARG;
    if (num_pages * PS + kTileKeys >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  }
  const int64_t grid = plan->units;
  if (grid != (int64_t)plan->q_tiles * plan->n_kv_heads * S || grid <= 0 ||
      grid >= (int64_t(1) << 31))
    return PA_ERR_INVALID_ARG;

  CUtensorMap tk, tv;
  const int64_t rows = paged ? num_pages * PS : total_keys;
  const int box_rows = paged ? PS : kTileKeys;
  if (!make_kv_map(&tk, k_pool, bf16, D, plan->n_kv_heads, rows, box_rows) ||
      !make_kv_map(&tv, v_pool, bf16, D, plan->n_kv_heads, rows, box_rows))
    return PA_ERR_CUDA;

  PrefillArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.page_table = page_table;
  a.out = out;
  a.ws_o = S > 1 ? lse_ws : nullptr;
  a.ws_lse = S > 1 ? lse_ws + (int64_t)S * chunk_rows * plan->n_q_heads * D : nullptr;
  a.hist_len = hist_len;
  a.table_len = paged ? (total_keys + PS - 1) / PS : 0;
  a.total_keys = total_keys;
  a.R = chunk_rows;
  a.Hq = plan->n_q_heads;
  a.Hkv = plan->n_kv_heads;
  a.G = plan->group;
  a.q_tiles = plan->q_tiles;
  a.splits = S;
  a.page_size = paged ? PS : 0;
  a.pages_per_tile = paged ? kTileKeys / PS : 1;
  a.num_pages = paged ? (int32_t)num_pages : 0;
  a.oob_row = (int32_t)rows;
  a.scale_log2 = plan->scale * 1.4426950408889634f;
  a.timeout_ns = g_timeout_ns.load();

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  switch (D) {
    case 64: e = launch_d<64>(paged, bf16, grid, st, tk, tv, a); break;
    case 128: e = launch_d<128>(paged, bf16, grid, st, tk, tv, a); break;
    default: e = launch_d<256>(paged, bf16, grid, st, tk, tv, a); break;
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_combine(const pa_plan_t* plan, const float* lse_ws, uint64_t ws_bytes,
                          float* out, pa_stream_t stream) {
  if (!plan) return PA_ERR_INVALID_ARG;
  const int S = plan->splits;
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
