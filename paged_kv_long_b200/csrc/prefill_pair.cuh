// prefill_pair.cuh — the head-dim-256 prefill kernel on CTA pairs (a cluster of two CTAs whose
// tensor cores work as one, tcgen05 cta_group::2). Included by pa_kernels.cu.
//
// A unit is (KV head, pair of packed Q tiles, history split) or a balanced work item. CTA rank
// r of the pair holds Q tile 2t+r (its own 128 rows): its Q in shared memory, its S, P and O
// in its own tensor memory, and its softmax warps. Rank 0 issues every MMA of the pair with
// M = 256:
//   S = Q K^T:  A = the two Q tiles (shared memory), B = K split by keys (rank r holds keys
//               64r..64r+63 of each 128-key tile, all 256 of D);
//   O += P V:   A = the two P tiles (tensor memory), B = V split by D (rank r holds dims
//               128r..128r+127 of all 128 keys).
// Each CTA therefore loads half of every K/V tile. Each CTA's copies fill its own shared
// memory, and both halves of a slot complete on rank 0's barrier (the pair form of the tensor
// copy), so rank 0 sees a slot as one unit; rank 0's MMA completions reach both CTAs
// (multicast commits).
//
// The tile loop. Tensor memory (512 columns) holds O (256), one S buffer (128) and two P
// buffers (64 columns of 16-bit pairs each). The softmax warps read S(j) into registers and
// release the buffer at once (s_free), so that QK(j+1) runs while the softmax of tile j does;
// P(j) goes to P buffer j % 2, which the softmax writes once PV(j-2) (its last reader) is
// done. Two threads of rank 0 issue the MMAs: one every QK, the other every PV.
// tcgen05.mma holds its issuing thread until the tensor pipe takes the instruction, so a
// single issuer leaves the pipe idle through every wait and commit between its MMA groups
// (measured: ~900 of ~3,100 cycles per tile); with two, one stream feeds the pipe while the
// other waits, and QK and PV (different accumulators) interleave. K and V land in rings of
// their own (three and two half tiles of 16 KB slots), each filled in tile order by a copy warp
// of its own: V(j) reuses the slots of V(j-2) (released when PV(j-2) completes), not those
// of a K half tile that QK(j) releases just before PV(j) needs V(j), which left V one tile
// of lookahead and made small pages (more boxes to issue per tile) land late.
//
// Rank 1's softmax warps announce the end of their S reads and their P to rank 0 with
// CTA-scope remote arrivals (tensor-memory accesses, ordered by tcgen05.wait and the
// before-thread-sync fence). Where they also wrote their CTA's shared memory (a Q tile loaded
// by the threads; V rows zeroed in the last tile) each thread makes the writes visible to the
// async proxy and releases them at cluster scope with a fence restricted to its own CTA's
// shared memory before a relaxed cluster-scope arrival (a full cluster-scope release measured
// ~1,400 cycles). The V rows of the sequence's last, partly filled tile complete on the
// issuing CTA's own barrier, because its softmax warps zero the rows past the end before the
// PV product reads them.

constexpr int kPairThreads = 256;    // warps: 0-3 softmax, 4 QK issuer, 5-6 copies, 7 PV issuer
constexpr int kPairPvWarp = 7;
constexpr int kPairIssuers = 2;      // copy-issuing warps
constexpr uint32_t kPairSCol = 256;  // S: one buffer of 128 columns
constexpr uint32_t kPairPCol = 384;  // P: buffers of 64 columns (16-bit pairs) at 384 and 448

struct PairCfg {
  static constexpr int NP = 4;        // 64-wide panels of a 256-wide row
  static constexpr int KSLOT = 6;     // K ring: 16 KB slots, a half tile is 2 slots
  static constexpr int VSLOT = 4;     // V ring (after the K ring)
  static constexpr int NSLOT = KSLOT + VSLOT;
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NP * kPanel;
  static constexpr int BAR_OFF = RING_OFF + NSLOT * kPanel;
  // full[10] (rank 0: both halves landed), empty[10] (K ring slots 0-5, V ring 6-9), q_full,
  // s_full, s_free, p_full[2], pv_done[2], mma_done (both issuers' last commits), teardown
  static constexpr int B_FULL = 0, B_EMPTY = NSLOT, B_QFULL = 2 * NSLOT,
                       B_SFULL = 2 * NSLOT + 1, B_SFREE = 2 * NSLOT + 2, B_PFULL = 2 * NSLOT + 3,
                       B_PVDONE = 2 * NSLOT + 5, B_MMADONE = 2 * NSLOT + 7,
                       B_TEAR = 2 * NSLOT + 8, N_BARS = 2 * NSLOT + 9;
  static constexpr int MISC_OFF = BAR_OFF + 8 * N_BARS;
  static constexpr int SMEM = MISC_OFF + 16;
  static constexpr int LAUNCH_SMEM = SMEM + 1024;
  static_assert(LAUNCH_SMEM <= 232448, "exceeds 227 KB of shared memory per CTA");
  // the epilogue stages 128 rows of 1 KB (+16 B) over the ring, idle by then
  static_assert(NSLOT * kPanel >= kTileRows * (256 * 4 + 16), "staging needs the ring");
};

// Byte offset inside a V half tile (2 slots: keys 0-63, then 64-127) of key row k, local panel
// pl (0 or 1): boxes of v_rows keys x 2 panels, panel after panel.
__device__ __forceinline__ uint32_t v_offset_pair(uint32_t k, uint32_t pl, int v_shift) {
  const uint32_t kk = k & 63u;
  return ((k >> 6) << 14) + ((kk >> v_shift) << (v_shift + 8)) + ((pl << v_shift) << 7) +
         ((kk & ((1u << v_shift) - 1u)) << 7);
}

// Fill q of a ring (half tile q / 2, slot half q % 2): K fill q sits in slot q % KSLOT, V fill
// q in slot KSLOT + q % VSLOT; a fill has landed when phase (q / ring size) % 2 of its slot's
// full barrier completes.
__device__ __forceinline__ uint32_t pair_k_slot(uint32_t q) { return q % PairCfg::KSLOT; }
__device__ __forceinline__ uint32_t pair_k_phase(uint32_t q) { return (q / PairCfg::KSLOT) & 1u; }
__device__ __forceinline__ uint32_t pair_v_slot(uint32_t q) {
  return PairCfg::KSLOT + q % PairCfg::VSLOT;
}
__device__ __forceinline__ uint32_t pair_v_phase(uint32_t q) { return (q / PairCfg::VSLOT) & 1u; }

// Barriers of the pair's softmax warps besides those of SoftmaxCtx.
struct PairSync {
  uint32_t arrive_sfree;  // s_free of rank 0 (remote on rank 1)
  uint32_t arrive_p;      // p_full[0] of rank 0 (remote on rank 1); +8: buffer 1
};

// Softmax + epilogue warps of the pair kernel (warps 0-3, one thread per packed Q row of this
// CTA's tile = tensor-memory lane).
template <bool PAGED, bool BF16, class VTail>
__device__ __forceinline__ void softmax_pair_role(const PrefillArgs& a, const SoftmaxCtx& x,
                                                  const PairSync& y, VTail&& v_tail) {
  constexpr int D = 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tmem = x.tmem;
  const int64_t qt = x.qt, kt0 = x.kt0;
  const int g = x.g, n = x.n;
  volatile int* abort_flag = x.abort_flag;
  const uint64_t tmo = x.tmo;
  const int r = threadIdx.x;  // packed Q row = tensor-memory lane
  const int64_t grow = qt * kTileRows + r;
  const int64_t tok = grow / a.G;
  const bool valid = tok < a.R;
  const int head = g * a.G + (int)(grow % a.G);
  const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
  if (!a.q_tma) {
    // Q tile -> shared memory as K-major rows of 64-element panels, 128-byte swizzle (when the
    // tensor copy cannot: it loads whole tokens, so it needs G to divide 128).
    const uint4* src =
        reinterpret_cast<const uint4*>(a.q + (valid ? (tok * a.Hq + head) * (int64_t)D : 0));
#pragma unroll
    for (int p = 0; p < 4; ++p) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = valid ? __ldg(src + p * 8 + c) : make_uint4(0u, 0u, 0u, 0u);
        st_shared_v4(x.sb + x.q_off + p * kPanel + r * 128 + ((c ^ (r & 7)) << 4), v.x, v.y,
                     v.z, v.w);
      }
    }
    fence_proxy_async_smem();
    if (x.remote_arrive) fence_release_smem_cluster();
    __syncwarp();
    if (lane == 0) {
      if (x.remote_arrive)
        mbar_arrive_remote_relaxed(x.arrive_qfull);
      else
        mbar_arrive(x.arrive_qfull);
    }
  }

  const int64_t limit = valid ? a.hist_len + tok : -1;  // last key this row may see
  const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
  float m_run = -INFINITY;  // running max of scale*log2(e)*score
  float l_run = 0.f;        // running sum of the probabilities (fp32)
  bool ok = true;
  // PV of tile i completes phase (i / 2) % 2 of pv_done[i % 2]. The softmax waits for PV(i)
  // only at tiles i + 1 (a rescale of O) and i + 2 (P's buffer); the next completion on that
  // barrier, PV(i + 2), needs P(i + 2), stored after those waits, so no parity wait skips a
  // phase.
  auto wait_pv = [&](int i) -> bool {
    return warp_wait(x.bar_pvdone + 8u * (uint32_t)(i & 1), (uint32_t)(i >> 1) & 1u, abort_flag,
                     tmo);
  };
  for (int j = 0; j < n; ++j) {
    const int64_t key0 = (kt0 + j) * kTileKeys;
    if (!warp_wait(x.bar_sfull, (uint32_t)j & 1u, abort_flag, tmo)) {
      ok = false;
      break;
    }
    tc_fence_after();
    float sv[kTileKeys];
#pragma unroll
    for (int c = 0; c < kTileKeys / 32; ++c)
      tmem_ld32(t_lane + kPairSCol + 32u * c, *reinterpret_cast<float(*)[32]>(&sv[32 * c]));
    tmem_wait_ld();
    // S(j) is in registers: the buffer may take S(j+1)
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (x.remote_arrive)
        mbar_arrive_remote_tc(y.arrive_sfree);
      else
        mbar_arrive(y.arrive_sfree);
    }

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
    // The probabilities use the new reference whenever it moves; O (and l) are brought to it
    // below, once the PV that last wrote O has completed.
    const float f_resc = (need && m_run != -INFINITY) ? ex2(m_run - m_new) : 1.0f;
    if (need) m_run = m_new;
    const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
    const float2 nm2 = make_float2(-m_use, -m_use);
    float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                    make_float2(0.f, 0.f)};
    uint32_t pk[kTileKeys / 2];
#pragma unroll
    for (int c = 0; c < kTileKeys; c += 2) {
      const float2 t = ffma2(make_float2(sv[c], sv[c + 1]), sc2, nm2);
      const float2 pr = make_float2(ex2(t.x), ex2(t.y));
      ls[(c >> 1) & 3] = fadd2(ls[(c >> 1) & 3], pr);
      pk[c >> 1] = pack2<BF16>(pr.x, pr.y);
    }
    const float l_tile = (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y) + (ls[2].x + ls[2].y) +
                         (ls[3].x + ls[3].y);
    if (j >= 1 && __any_sync(0xffffffffu, f_resc != 1.0f)) {
      // O must not change under a running MMA: wait for PV(j-1), the last to write it
      if (!wait_pv(j - 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(t_lane + kOCol + 32u * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] *= f_resc;
        tmem_st32(t_lane + kOCol + 32u * c, o);
      }
      tmem_wait_st();
    }
    l_run = l_run * f_resc + l_tile;
    // P's buffer j % 2 was last read by PV(j-2)
    if (j >= 2 && !wait_pv(j - 2)) {
      ok = false;
      break;
    }

    // The sequence's last tile, partly past its end (paged pools): this CTA's half of the V
    // rows past the end is zeroed in shared memory before PV reads it.
    const bool tail = PAGED && key0 + kTileKeys > a.total_keys;
    if (tail && !v_tail(j, key0 + r >= a.total_keys ? r : -1)) {
      ok = false;
      break;
    }
    // P(j) (rounded to the input type) into P buffer j % 2: one row per lane, 16-bit pairs
    const uint32_t p_col = kPairPCol + 64u * (uint32_t)(j & 1);
    tmem_st32u(t_lane + p_col, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
    tmem_st32u(t_lane + p_col + 32u, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
    tmem_wait_st();
    tc_fence_before();
    if (tail) {
      fence_proxy_async_smem();
      if (x.remote_arrive) fence_release_smem_cluster();
    }
    __syncwarp();
    if (lane == 0) {
      const uint32_t pb = y.arrive_p + 8u * (uint32_t)(j & 1);
      if (!x.remote_arrive)
        mbar_arrive(pb);
      else if (tail)
        mbar_arrive_remote_relaxed(pb);
      else
        mbar_arrive_remote_tc(pb);
    }
  }

  if (ok && n >= 2) ok = wait_pv(n - 2);
  if (ok) ok = wait_pv(n - 1);
  if (ok) {
    tc_fence_after();
    write_row<D>(a, x, r, valid, tok, head, m_run, l_run, t_lane);
  }
}

template <bool PAGED, bool BF16>
__global__ void __launch_bounds__(kPairThreads, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const PrefillArgs a_in,
                        const __grid_constant__ ItemTable items) {
  PrefillArgs a = a_in;  // rebased on one sequence in batched plans
  using C = PairCfg;
  constexpr int D = 256, NSLOT = C::NSLOT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 issues the MMAs

  int64_t tp, kt0, kt1;
  int g, s, slot = kSlotUniform;
  if (a.balanced) {
    const PaItem it = items.item[blockIdx.x >> 1];
    const int32_t rb = a.batch > 0 ? batch_rebase<D>(a, items, it.rb) : it.rb;
    rb_coords(rb, (a.q_tiles + 1) / 2, a.Hkv, &tp, &g);
    s = 0;
    kt0 = it.kt0;
    kt1 = it.kt1;
    slot = it.slot;
  } else {
    unit_coords(blockIdx.x >> 1, (a.q_tiles + 1) / 2, a.Hkv, a.splits, &tp, &g, &s);
    const int64_t qt_last = 2 * tp + 1 < a.q_tiles ? 2 * tp + 1 : a.q_tiles - 1;
    split_range(tile_kv_tiles(qt_last, a.R, a.G, a.hist_len), s, a.splits, &kt0, &kt1);
  }
  const int64_t qt = 2 * tp + rank;
  const int n = (int)(kt1 - kt0);

  if (n == 0) {  // both CTAs of the pair see the same (empty) key range: empty partial
    if (threadIdx.x < kTileRows) {
      const int64_t grow = qt * kTileRows + threadIdx.x;
      const int64_t tok = grow / a.G;
      if (tok < a.R) {
        const int head = g * a.G + (int)(grow % a.G);
        const int64_t row = (int64_t)s * a.ws_split_rows + tok * a.Hq + head;
        float4* d4 = reinterpret_cast<float4*>(a.ws_o + row * D);
        for (int i = 0; i < D / 4; ++i) d4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        a.ws_lse[row] = -INFINITY;
      }
    }
    return;
  }

  // The copy warps read the page-table entries of the first two KV tiles before the set-up
  // below, so the loads overlap it and the first copies go out right after it.
  int32_t pre_row0 = a.oob_row, pre_row1 = a.oob_row;
  if (warp > kMmaWarp && warp < kPairPvWarp) {
    const bool report = warp == kMmaWarp + 1;
    pre_row0 = tile_page_row<PAGED>(a, kt0, n, 0, lane, report);
    pre_row1 = tile_page_row<PAGED>(a, kt0, n, 1, lane, report);
  }
  auto bar = [&](int i) -> uint32_t { return sb + C::BAR_OFF + 8u * (uint32_t)i; };
  auto slot_addr = [&](uint32_t slot) -> uint32_t { return sb + C::RING_OFF + slot * kPanel; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF + 4);
  const uint32_t leader_bar0 = mapa_shared(sb + C::BAR_OFF, 0);  // rank 0's barriers
  auto leader_bar = [&](int i) -> uint32_t { return leader_bar0 + 8u * (uint32_t)i; };
  // The sequence's last KV tile, partly past the end (paged pools only: there the rows after
  // the last key hold another sequence's data or nothing), is the unit's last tile; its V
  // fills are the V ring's last two (2n-2, 2n-1).
  const bool has_tail = PAGED && (kt0 + n) * kTileKeys > a.total_keys;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(bar(C::B_FULL + i), 1);
      mbar_init(bar(C::B_EMPTY + i), 1);
    }
    // Q by tensor copy: one arrival (rank 0's, with both CTAs' bytes); else 4 softmax warps
    // here + 4 of rank 1
    mbar_init(bar(C::B_QFULL), a.q_tma ? 1 : 8);
    mbar_init(bar(C::B_SFULL), 1);
    mbar_init(bar(C::B_SFREE), 8);      // 4 softmax warps here + 4 of rank 1
    mbar_init(bar(C::B_PFULL + 0), 8);  // 4 softmax warps here + 4 of rank 1
    mbar_init(bar(C::B_PFULL + 1), 8);
    mbar_init(bar(C::B_PVDONE + 0), 1);
    mbar_init(bar(C::B_PVDONE + 1), 1);
    mbar_init(bar(C::B_MMADONE), 2);
    mbar_init(bar(C::B_TEAR), 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp + 1 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (a.q_tma) tma_prefetch_desc(&tm_q);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;

  // Cluster-scope bounded wait (for barriers the other CTA arrives on).
  auto wait_cluster = [&](uint32_t b, uint32_t parity) -> bool {
    if (mbar_try_wait_cluster(b, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_wait_cluster(b, parity)) return true;
      if ((it & 31u) == 0) {
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > tmo) {
          *abort_flag = 1;
          atomicOr(&g_pa_error_flags, kFlagTimeout);
          return false;
        }
      }
    }
  };

  if (warp < 4) {
    // ============================================================ softmax + epilogue
    SoftmaxCtx sc;
    sc.sb = sb;
    sc.q_off = C::Q_OFF;
    sc.bar_sfull = bar(C::B_SFULL);
    sc.bar_pvdone = bar(C::B_PVDONE);
    sc.remote_arrive = rank != 0;
    sc.arrive_qfull = rank == 0 ? bar(C::B_QFULL) : leader_bar(C::B_QFULL);
    sc.arrive_pfull = 0;
    sc.tmem = tmem;
    sc.qt = qt;
    sc.g = g;
    sc.s = s;
    sc.kt0 = kt0;
    sc.n = n;
    sc.slot = slot;
    sc.row0 = (int)rank * kTileRows;
    sc.stage_off = C::RING_OFF;
    sc.abort_flag = abort_flag;
    sc.tmo = tmo;
    PairSync ps;
    ps.arrive_sfree = rank == 0 ? bar(C::B_SFREE) : leader_bar(C::B_SFREE);
    ps.arrive_p = rank == 0 ? bar(C::B_PFULL) : leader_bar(C::B_PFULL);
    // Keys past the sequence in its last page hold arbitrary bits; P is 0 there but 0 * NaN
    // is NaN inside the MMA, so this CTA's half of those V rows is zeroed before PV.
    // Those fills complete on this CTA's own barrier: on rank 1 that barrier sees no other
    // phase, so its parity is 0.
    auto v_tail = [&](int j, int r) -> bool {
      const uint32_t seq0 = 2u * (uint32_t)j;
      bool okv = true;
      for (int k = 0; k < 2 && okv; ++k)
        okv = warp_wait(bar(C::B_FULL + pair_v_slot(seq0 + k)),
                        rank == 0 ? pair_v_phase(seq0 + k) : 0u, abort_flag, tmo);
      if (!okv || r < 0) return okv;
      for (int pl = 0; pl < 2; ++pl) {
        const uint32_t off = v_offset_pair((uint32_t)r, pl, a.v_shift);
        const uint32_t ra = slot_addr(pair_v_slot(seq0 + (off >> 14))) + (off & (kPanel - 1));
#pragma unroll
        for (int c = 0; c < 8; ++c) st_shared_v4(ra + c * 16, 0u, 0u, 0u, 0u);
      }
      return true;
    };
    softmax_pair_role<PAGED, BF16>(a, sc, ps, v_tail);
  } else if (warp > kMmaWarp && warp < kPairPvWarp) {
    // ============================================================ TMA issuers (two warps)
    // Warp 5 fills the K ring (K(0), K(1), ... in tile order), warp 6 the V ring; lanes issue
    // one box each.
    const int w = warp - kMmaWarp - 1;
    const int ppt = a.pages_per_tile;
    const int prow = a.page_rows;
    const int k_rows = a.k_rows;                 // key rows per K box (<= 64)
    const int k_per_panel = 64 / k_rows;         // K boxes per (half tile, panel)
    const int v_rows = 1 << a.v_shift;           // key rows per V box (<= 64)
    const int v_per_slot = 64 / v_rows;
    bool ok = true;
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
    // Key-row coordinate of key kk (0..127) of a tile whose page rows sit in `rows` (lane i:
    // page i). All lanes take part in the shuffle.
    auto key_row = [&](int32_t rows, int kk) -> int32_t {
      const int pg = kk >> a.page_shift;
      const int32_t base = __shfl_sync(0xffffffffu, rows, pg & 31);
      return base == a.oob_row ? a.oob_row : base + (kk & (prow - 1));
    };
    // Wait until a slot is free for its `use`-th fill and announce the bytes. Rank 0 expects
    // both halves of a slot on its barrier; rank 1 arms its own barrier only for the tail fills.
    auto acquire = [&](uint32_t slot, uint32_t use, bool tail) -> bool {
      bool r_ok =
          use == 0 || warp_wait(bar(C::B_EMPTY + slot), (use - 1) & 1, abort_flag, tmo);
      if (r_ok && lane == 0) {
        if (rank == 0) mbar_arrive_expect_tx(bar(C::B_FULL + slot), tail ? kPanel : 2 * kPanel);
        else if (tail) mbar_arrive_expect_tx(bar(C::B_FULL + slot), kPanel);
      }
      __syncwarp();
      return r_ok;
    };
    uint32_t issued = 0;  // fills this warp issued
    // K half tile m (keys 64*rank..+63 of tile m, all of D) in two slots. Per-panel boxes: slot
    // k holds panels 2k, 2k+1 (64 keys each). Atom boxes (a.k_atoms): box i = keys 8i..8i+7 x
    // all four panels (4 KB, panel after panel) at 4 KB * i from the first slot, boxes 4k..4k+3
    // in slot k; the half tile's two slots are adjacent (KSLOT is even).
    auto issue_k = [&](int m, int32_t rows) {
      for (int k = 0; k < 2 && ok; ++k) {
        const uint32_t q = 2u * (uint32_t)m + (uint32_t)k;
        const uint32_t sl = pair_k_slot(q);
        if (a.k_atoms) {
          const int32_t row = key_row(rows, 64 * (int)rank + 8 * (4 * k + (lane & 3)));
          if (!(ok = acquire(sl, q / C::KSLOT, false))) break;
          if (lane < 4) {
            const uint32_t dst = slot_addr(sl) + (uint32_t)lane * 4096u;
            if (rank == 0)
              tma_load_4d(dst, &tm_k, bar(C::B_FULL + sl), 0, row, 0, g);
            else
              tma_load_4d_pair(dst, &tm_k, leader_bar(C::B_FULL + sl), 0, row, 0, g);
          }
        } else {
          const int l = lane, pl = l / k_per_panel, sub = l - pl * k_per_panel;
          const int32_t row = key_row(rows, 64 * (int)rank + sub * k_rows);
          if (!(ok = acquire(sl, q / C::KSLOT, false))) break;
          if (l < 2 * k_per_panel) {
            const uint32_t dst = slot_addr(sl) + pl * (kPanel / 2) + sub * k_rows * 128;
            if (rank == 0)
              tma_load_3d(dst, &tm_k, bar(C::B_FULL + sl), (2 * k + pl) * 64, g, row);
            else
              tma_load_3d_pair(dst, &tm_k, leader_bar(C::B_FULL + sl), (2 * k + pl) * 64, g,
                               row);
          }
        }
        issued = q + 1;
      }
    };
    // V half tile j (dims 128*rank..+127 of tile j): slot k holds keys 64k..64k+63
    auto issue_v = [&](int j, int32_t rows) {
      const bool tail = has_tail && j == n - 1;
      for (int k = 0; k < 2 && ok; ++k) {
        const uint32_t q = 2u * (uint32_t)j + (uint32_t)k;
        const int32_t row = key_row(rows, 64 * k + lane * v_rows);
        const uint32_t sl = pair_v_slot(q);
        if (!(ok = acquire(sl, q / C::VSLOT, tail))) break;
        if (lane < v_per_slot) {
          const uint32_t dst = slot_addr(sl) + lane * (v_rows * 256);
          if (rank == 0 || tail)
            tma_load_4d(dst, &tm_v, bar(C::B_FULL + sl), 0, row, 2 * (int)rank, g);
          else
            tma_load_4d_pair(dst, &tm_v, leader_bar(C::B_FULL + sl), 0, row, 2 * (int)rank, g);
        }
        issued = q + 1;
      }
    };
    // Q tile: four 16 KB panels of 128/G whole tokens; both CTAs' bytes complete on rank 0's
    // barrier, which rank 0 arms for both. Rows past the piece arrive as zeros.
    if (a.q_tma && w == 0 && lane == 0) {
      const int32_t t0 = a.q_row0 + (int32_t)(qt * (kTileRows / a.G));
      if (rank == 0) mbar_arrive_expect_tx(bar(C::B_QFULL), 2u * 4u * kPanel);
      for (int p = 0; p < 4; ++p) {
        if (rank == 0)
          tma_load_4d(sb + C::Q_OFF + p * kPanel, &tm_q, bar(C::B_QFULL), p * 64, 0, g, t0);
        else
          tma_load_4d_pair(sb + C::Q_OFF + p * kPanel, &tm_q, leader_bar(C::B_QFULL), p * 64, 0,
                           g, t0);
      }
    }
    // Page rows of tiles t .. t+3 (lane i: page i of the tile); the rows of tile t+4 are loaded
    // while tile t is issued, three tiles before they are used.
    int32_t row_0 = pre_row0, row_1 = pre_row1, row_2 = fetch(2), row_3 = fetch(3);
    for (int t = 0; t < n && ok; ++t) {
      if (w == 0)
        issue_k(t, row_0);
      else
        issue_v(t, row_0);
      row_0 = row_1;
      row_1 = row_2;
      row_2 = row_3;
      row_3 = fetch(t + 4);
    }
    // Wait for this warp's last copies of each slot. On rank 0 the barrier covers both halves,
    // so rank 1's copies have landed as well; rank 1 drains only the tail fills on its own
    // barrier, and it stays resident until rank 0 has finished (teardown handshake below).
    const uint32_t ring = w == 0 ? C::KSLOT : C::VSLOT;
    for (uint32_t q = issued > ring ? issued - ring : 0; q < issued; ++q) {
      const bool tail = w == 1 && has_tail && q + 2u >= 2u * (uint32_t)n;
      if (rank == 0 || tail)
        drain_wait(bar(C::B_FULL + (w == 0 ? pair_k_slot(q) : pair_v_slot(q))),
                   rank == 0 ? (w == 0 ? pair_k_phase(q) : pair_v_phase(q)) : 0u, abort_flag,
                   tmo);
    }
    __syncwarp();
  } else if (rank == 0) {
    // ============================================================ MMA issuers (rank 0)
    // warp 4 lane 0 issues every QK, warp 7 lane 0 every PV; each commits only its own MMAs
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_f16(256, kTileKeys, BF16, false);
      constexpr uint32_t idesc_pv = umma_idesc_f16(256, D, BF16, true);
      constexpr uint32_t kSlotDesc = kPanel >> 4;
      constexpr uint16_t kBoth = 0x3;
      // a fill has landed (one barrier for both halves; for the tail fills rank 1's half is
      // covered by its softmax warps' P arrival, which they give after waiting for it)
      auto wait_fill = [&](uint32_t slot, uint32_t phase) -> bool {
        return thread_wait(bar(C::B_FULL + slot), phase, abort_flag, tmo);
      };
      bool ok = true;
      if (warp == kMmaWarp) {
        const uint64_t q_desc = smem_desc_sw128(sb + C::Q_OFF, 16, 1024);
        const uint64_t k_desc = smem_desc_sw128(sb + C::RING_OFF, 16, 1024);
        const uint32_t s_tmem = tmem + kPairSCol;
        // S(m) = Q K(m)^T into the S buffer once the softmax has read S(m-1): slot k of the K
        // half tile holds D panels 2k and 2k+1 (Q panels 2k, 2k+1). S(m) is completion m of
        // s_full and the read of S(m) arrival m of s_free.
        // Atom boxes: panel p of the half tile starts 1 KB * p into its first slot, its 8-key
        // atoms 4 KB apart across both slots, which are waited for first and released after
        // all four panels.
        const uint64_t k_desc_atoms = smem_desc_sw128(sb + C::RING_OFF, 16, 4096);
        ok = wait_cluster(bar(C::B_QFULL), 0);
        for (int m = 0; m < n && ok; ++m) {
          if (m >= 1) ok = wait_cluster(bar(C::B_SFREE), (uint32_t)(m - 1) & 1u);
          const uint32_t q0 = 2u * (uint32_t)m;
          if (a.k_atoms) {
            const uint32_t sl0 = pair_k_slot(q0), sl1 = pair_k_slot(q0 + 1);
            if (ok) ok = wait_fill(sl0, pair_k_phase(q0));
            if (ok) ok = wait_fill(sl1, pair_k_phase(q0 + 1));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const uint64_t ad = q_desc + p * kSlotDesc;
              const uint64_t bd = k_desc_atoms + sl0 * kSlotDesc + p * (1024 >> 4);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_ss_pair(s_tmem, ad + 2 * ks, bd + 2 * ks, idesc_qk, (p | ks) != 0 ? 1u : 0u);
            }
            umma_commit_pair(bar(C::B_EMPTY + sl0), kBoth);
            umma_commit_pair(bar(C::B_EMPTY + sl1), kBoth);
            umma_commit_pair(bar(C::B_SFULL), kBoth);
            continue;
          }
#pragma unroll
          for (int k = 0; k < 2 && ok; ++k) {
            if (!(ok = wait_fill(pair_k_slot(q0 + k), pair_k_phase(q0 + k)))) break;
            tc_fence_after();
            const uint32_t sl = pair_k_slot(q0 + k);
#pragma unroll
            for (int pl = 0; pl < 2; ++pl) {
              const int p = 2 * k + pl;
              const uint64_t ad = q_desc + p * kSlotDesc;
              const uint64_t bd = k_desc + sl * kSlotDesc + pl * (kSlotDesc / 2);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_ss_pair(s_tmem, ad + 2 * ks, bd + 2 * ks, idesc_qk, (p | ks) != 0 ? 1u : 0u);
            }
            umma_commit_pair(bar(C::B_EMPTY + sl), kBoth);
          }
          if (ok) umma_commit_pair(bar(C::B_SFULL), kBoth);
        }
      } else {
        const uint64_t v_desc =
            smem_desc_sw128(sb + C::RING_OFF, (uint32_t)(1 << a.v_shift) * 128u, 1024);
        // O += P(i) V(i) once P(i) is stored (phase (i / 2) % 2 of p_full[i % 2]): each half of
        // the V tile (keys 0-63, then 64-127) against the matching columns of P(i)'s buffer
        // (16 keys = 8 columns), released after its 4 MMAs; PV(i) completes phase (i / 2) % 2
        // of pv_done[i % 2]
        for (int i = 0; i < n && ok; ++i) {
          ok = wait_cluster(bar(C::B_PFULL + (i & 1)), (uint32_t)(i >> 1) & 1u);
          const uint32_t p_tmem = tmem + kPairPCol + 64u * (uint32_t)(i & 1);
          const uint32_t q0 = 2u * (uint32_t)i;
#pragma unroll
          for (int h = 0; h < 2 && ok; ++h) {
            if (!(ok = wait_fill(pair_v_slot(q0 + h), pair_v_phase(q0 + h)))) break;
            tc_fence_after();
            const uint32_t sl = pair_v_slot(q0 + h);
#pragma unroll
            for (int ks = 4 * h; ks < 4 * h + 4; ++ks) {
              const uint32_t off = v_offset_pair(16u * ks, 0, a.v_shift);
              umma_ts_pair(tmem + kOCol, p_tmem + (uint32_t)ks * 8u,
                           v_desc + sl * kSlotDesc + ((off & (kPanel - 1)) >> 4), idesc_pv,
                           (i > 0 || ks > 0) ? 1u : 0u);
            }
            umma_commit_pair(bar(C::B_EMPTY + sl), kBoth);
          }
          if (ok) umma_commit_pair(bar(C::B_PVDONE + (i & 1)), kBoth);
        }
      }
      // every MMA of both issuers must finish before tensor memory is freed
      umma_commit_pair(bar(C::B_MMADONE), kBoth);
      drain_wait(bar(C::B_MMADONE), 0, abort_flag, tmo);
    }
    __syncwarp();
  } else {
    // ============================================================ rank 1, MMA warps
    // rank 0's last MMAs have read this CTA's shared and tensor memory
    if (lane == 0) drain_wait(bar(C::B_MMADONE), 0, abort_flag, tmo);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    // The pair's tensor memory is freed only when both CTAs are done with it.
    if (lane == 0) mbar_arrive_remote(mapa_shared(bar(C::B_TEAR), rank ^ 1u));
    __syncwarp();
    if (lane == 0 && !mbar_try_wait_cluster(bar(C::B_TEAR), 0)) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait_cluster(bar(C::B_TEAR), 0))
        if (globaltimer_ns() - t0 > tmo) {
          atomicOr(&g_pa_error_flags, kFlagTimeout);
          break;
        }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}
