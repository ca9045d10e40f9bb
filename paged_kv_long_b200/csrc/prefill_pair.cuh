// prefill_pair.cuh — the head-dim-256 prefill kernel on CTA pairs (a cluster of two CTAs whose
// tensor cores work as one, tcgen05 cta_group::2). Included by pa_kernels.cu.
//
// A unit is (KV head, pair of packed Q tiles, history split). CTA rank r of the pair holds
// Q tile 2t+r (its own 128 rows): its Q in shared memory, its S/P and O in its own tensor
// memory, and its softmax warps. Rank 0 issues every MMA of the pair with M = 256:
//   S = Q K^T:  A = the two Q tiles, B = K split by keys (rank r holds keys 64r..64r+63 of
//               each 128-key tile, all 256 of D);
//   O += P V:   A = the two P tiles (each in its own tensor memory), B = V split by D (rank r
//               holds dims 128r..128r+127 of all 128 keys).
// Each CTA therefore loads half of every K/V tile: half the L2 traffic per FLOP of the
// single-CTA kernel, and twice the time its shared-memory ring covers. Each CTA's copies fill
// its own shared memory, and both halves of a slot complete on rank 0's barrier (the pair form
// of the tensor copy), so rank 0 sees a slot as one unit. Rank 1 tells rank 0 when its Q and P
// are ready (remote mbarrier arrivals); rank 0's MMA completions reach both CTAs (multicast
// commits). One exception: the V rows of the sequence's last, partly filled tile complete on
// the issuing CTA's own barrier, because its softmax warps zero the rows past the end before
// the PV product reads them.

struct PairCfg {
  static constexpr int NP = 4;        // 64-wide panels of a 256-wide row
  static constexpr int NSLOT = 10;    // ring of 16 KB slots; a half tile (K or V) is 2 slots
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = NP * kPanel;
  static constexpr int BAR_OFF = RING_OFF + NSLOT * kPanel;
  // full[10] (rank 0: both halves landed), empty[10], q_full, s_full[2], p_full[2],
  // pv_done[2], mma_done, teardown
  static constexpr int B_FULL = 0, B_EMPTY = NSLOT, B_QFULL = 2 * NSLOT,
                       B_SFULL = 2 * NSLOT + 1, B_PFULL = 2 * NSLOT + 3, B_PVDONE = 2 * NSLOT + 5,
                       B_MMADONE = 2 * NSLOT + 7, B_TEAR = 2 * NSLOT + 8, N_BARS = 2 * NSLOT + 9;
  static constexpr int MISC_OFF = BAR_OFF + 8 * N_BARS;
  static constexpr int SMEM = MISC_OFF + 16;
  static constexpr int LAUNCH_SMEM = SMEM + 1024;
  static_assert(LAUNCH_SMEM <= 232448, "exceeds 227 KB of shared memory per CTA");
};

// Byte offset inside a V half tile (2 slots: keys 0-63, then 64-127) of key row k, local panel
// pl (0 or 1): boxes of v_rows keys x 2 panels, panel after panel.
__device__ __forceinline__ uint32_t v_offset_pair(uint32_t k, uint32_t pl, int v_shift) {
  const uint32_t kk = k & 63u;
  return ((k >> 6) << 14) + ((kk >> v_shift) << (v_shift + 8)) + ((pl << v_shift) << 7) +
         ((kk & ((1u << v_shift) - 1u)) << 7);
}

template <bool PAGED, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
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
  PA_UNIT_ONLY(const uint64_t t_entry = globaltimer_ns(); const long long c_entry = clock64();)

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
  if (warp > kMmaWarp) {
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
  // fills are the unit's last two (4n-2, 4n-1).
  const bool has_tail = PAGED && (kt0 + n) * kTileKeys > a.total_keys;
  auto tail_fill = [&](uint32_t q) -> bool { return has_tail && q + 2u >= 4u * (uint32_t)n; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(bar(C::B_FULL + i), 1);
      mbar_init(bar(C::B_EMPTY + i), 1);
    }
    // Q by tensor copy: one arrival (rank 0's, with both CTAs' bytes); else 4 softmax warps
    // here + 4 of rank 1
    mbar_init(bar(C::B_QFULL), a.q_tma ? 1 : 8);
    mbar_init(bar(C::B_SFULL + 0), 1);
    mbar_init(bar(C::B_SFULL + 1), 1);
    mbar_init(bar(C::B_PFULL + 0), 8);
    mbar_init(bar(C::B_PFULL + 1), 8);
    mbar_init(bar(C::B_PVDONE + 0), 1);
    mbar_init(bar(C::B_PVDONE + 1), 1);
    mbar_init(bar(C::B_MMADONE), 1);
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
  PA_UNIT_ONLY(if (threadIdx.x == 0 && blockIdx.x < 8192)
                   g_pa_units[kUnitWords * blockIdx.x + 4] = clock64();)
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;
  PA_TRACE_ONLY(unsigned tln = 0;)

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
    sc.arrive_pfull = rank == 0 ? bar(C::B_PFULL) : leader_bar(C::B_PFULL);
    sc.tmem = tmem;
    sc.qt = qt;
    sc.g = g;
    sc.s = s;
    sc.kt0 = kt0;
    sc.n = n;
    sc.slot = slot;
    sc.row0 = (int)rank * kTileRows;
    sc.stage_off = C::RING_OFF;
    static_assert(NSLOT * kPanel >= kTileRows * (D * 4 + 16), "staging needs the ring");
    sc.abort_flag = abort_flag;
    sc.tmo = tmo;
    // Keys past the sequence in its last page hold arbitrary bits; P is 0 there but 0 * NaN
    // is NaN inside the MMA, so this CTA's half of those V rows is zeroed before PV.
    // Those fills complete on this CTA's own barrier: on rank 1 that barrier sees no other
    // phase, so its parity is 0.
    auto v_tail = [&](int j, int r) -> bool {
      const uint32_t seq0 = v_item(j, n) * 2;
      bool okv = true;
      for (int k = 0; k < 2 && okv; ++k)
        okv = warp_wait(bar(C::B_FULL + (seq0 + k) % NSLOT),
                        rank == 0 ? ((seq0 + k) / NSLOT) & 1 : 0u, abort_flag, tmo);
      if (!okv || r < 0) return okv;
      for (int pl = 0; pl < 2; ++pl) {
        const uint32_t off = v_offset_pair((uint32_t)r, pl, a.v_shift);
        const uint32_t ra = slot_addr((seq0 + (off >> 14)) % NSLOT) + (off & (kPanel - 1));
#pragma unroll
        for (int c = 0; c < 8; ++c) st_shared_v4(ra + c * 16, 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      return true;
    };
    softmax_role<D, PAGED, BF16>(a, sc, v_tail);
  } else if (warp > kMmaWarp) {
    // ============================================================ TMA issuers (three warps)
    // Fill q (2 per K or V half tile, in the order K0, K1, V0, K2, V1, ...) is issued by warp
    // q % kIssuers; lanes issue one box each.
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
    // Rank 0 expects both halves of a slot on its barrier; rank 1 arms its own barrier only for
    // the tail fills.
    auto acquire = [&](uint32_t q) -> bool {
      const uint32_t slot = q % NSLOT;
      PA_TRACE_ONLY(if (lane == 0) tlog(w, tln, 15, q);)
      bool r_ok = q < (uint32_t)NSLOT ||
                  warp_wait(bar(C::B_EMPTY + slot), ((q / NSLOT) - 1) & 1, abort_flag, tmo);
      if (r_ok && lane == 0) {
        const bool tail = tail_fill(q);
        if (rank == 0) mbar_arrive_expect_tx(bar(C::B_FULL + slot), tail ? kPanel : 2 * kPanel);
        else if (tail) mbar_arrive_expect_tx(bar(C::B_FULL + slot), kPanel);
      }
      __syncwarp();
      return r_ok;
    };
    auto own_barrier = [&](uint32_t q) -> bool { return rank == 0 || tail_fill(q); };
    int32_t row_prev = a.oob_row, row_cur = pre_row0, row_next = pre_row1;
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
    uint32_t issued_end = 0;
    for (int j = 0; j <= n && ok; ++j) {
      if (j < n) {  // K half tile j: slot k holds panels 2k, 2k+1 of keys 64*rank..+63
        const uint32_t item = j == 0 ? 0u : 2u * j - 1u;
        for (int k = 0; k < 2 && ok; ++k) {
          const uint32_t q = item * 2 + k;
          const int l = lane, pl = l / k_per_panel, sub = l - pl * k_per_panel;
          const int32_t row = key_row(row_cur, 64 * (int)rank + sub * k_rows);
          if ((int)(q % kIssuers) != w) continue;
          if (!(ok = acquire(q))) break;
          const uint32_t slot = q % NSLOT;
          if (l < 2 * k_per_panel) {
            const uint32_t dst = slot_addr(slot) + pl * (kPanel / 2) + sub * k_rows * 128;
            if (own_barrier(q))
              tma_load_3d(dst, &tm_k, bar(C::B_FULL + slot), (2 * k + pl) * 64, g, row);
            else
              tma_load_3d_pair(dst, &tm_k, leader_bar(C::B_FULL + slot), (2 * k + pl) * 64, g,
                               row);
          }
          issued_end = q + 1;
          PA_UNIT_ONLY(if (q == 0 && lane == 0 && blockIdx.x < 8192)
                           g_pa_units[kUnitWords * blockIdx.x + 11] = clock64();)
          PA_TRACE_ONLY(if (lane == 0) tlog(w, tln, 1, q);)
        }
      }
      if (ok && j >= 1) {  // V half tile j-1: slot k holds keys 64k..64k+63, dims 128*rank..+127
        const uint32_t item = v_item(j - 1, n);
        for (int k = 0; k < 2 && ok; ++k) {
          const uint32_t q = item * 2 + k;
          const int32_t row = key_row(row_prev, 64 * k + lane * v_rows);
          if ((int)(q % kIssuers) != w) continue;
          if (!(ok = acquire(q))) break;
          const uint32_t slot = q % NSLOT;
          if (lane < v_per_slot) {
            const uint32_t dst = slot_addr(slot) + lane * (v_rows * 256);
            if (own_barrier(q))
              tma_load_4d(dst, &tm_v, bar(C::B_FULL + slot), 0, row, 2 * (int)rank, g);
            else
              tma_load_4d_pair(dst, &tm_v, leader_bar(C::B_FULL + slot), 0, row, 2 * (int)rank,
                               g);
          }
          issued_end = q + 1;
          PA_TRACE_ONLY(if (lane == 0) tlog(w, tln, 2, q);)
        }
      }
      row_prev = row_cur;
      row_cur = row_next;
      row_next = fetch(j + 2);
    }
    // Wait for this warp's copies among the last NSLOT fills (see the single-CTA kernel). On
    // rank 0 the barrier covers both halves, so rank 1's copies have landed as well; rank 1
    // drains only the tail fills on its own barrier, and it stays resident until rank 0 has
    // finished (teardown handshake below).
    const uint32_t all_fills = 4u * n;
    for (uint32_t q = all_fills > (uint32_t)NSLOT ? all_fills - NSLOT : 0; q < issued_end; ++q)
      if ((int)(q % kIssuers) == w && own_barrier(q))
        drain_wait(bar(C::B_FULL + q % NSLOT), rank == 0 ? (q / NSLOT) & 1 : 0u, abort_flag,
                   tmo);
    __syncwarp();
  } else if (rank == 0) {
    // ============================================================ MMA issuer (rank 0, one lane)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_f16(256, kTileKeys, BF16, false);
      constexpr uint32_t idesc_pv = umma_idesc_f16(256, D, BF16, true);
      constexpr uint32_t kSlotDesc = kPanel >> 4;
      constexpr uint16_t kBoth = 0x3;
      const uint64_t q_desc = smem_desc_sw128(sb + C::Q_OFF, 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(sb + C::RING_OFF, 16, 1024);
      const uint64_t v_desc =
          smem_desc_sw128(sb + C::RING_OFF, (uint32_t)(1 << a.v_shift) * 128u, 1024);
      uint32_t slot = 0, round = 0;
      PA_TRACE_ONLY(unsigned tln_w = 0;)
      // a slot is ready when both halves landed (one barrier; for the tail fills rank 1's half
      // is covered by its softmax warps' P-ready arrival, which waits for it)
      PA_UNIT_ONLY(long long w_k = 0, w_v = 0, w_p = 0; long long* w_sel = &w_k;)
      auto wait_slot = [&]() -> bool {
        PA_TRACE_ONLY(tlog(6, tln_w, 11, round * NSLOT + slot);)
        PA_UNIT_ONLY(const long long c0 = clock64();)
        const bool r = thread_wait(bar(C::B_FULL + slot), round & 1, abort_flag, tmo);
        PA_UNIT_ONLY(*w_sel += clock64() - c0;)
        PA_TRACE_ONLY(tlog(6, tln_w, 12, round * NSLOT + slot);)
        return r;
      };
      auto advance = [&]() {
        if (++slot == (uint32_t)NSLOT) {
          slot = 0;
          ++round;
        }
      };
      bool ok = wait_cluster(bar(C::B_QFULL), 0);
      PA_UNIT_ONLY(if (blockIdx.x < 8192) g_pa_units[kUnitWords * blockIdx.x + 8] = clock64();)
      tc_fence_after();
      for (int j = 0; j <= n && ok; ++j) {
        if (j < n) {
          const uint32_t s_tmem = tmem + kSCol0 + 128u * (j & 1);
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            PA_UNIT_ONLY(w_sel = &w_k;)
            if (!(ok = wait_slot())) break;
            PA_UNIT_ONLY(if (j == 0 && k == 0 && blockIdx.x < 8192)
                             g_pa_units[kUnitWords * blockIdx.x + 9] = clock64();)
            PA_TRACE_ONLY(tlog(3, tln, 3, round * NSLOT + slot);)
            tc_fence_after();
#pragma unroll
            for (int pl = 0; pl < 2; ++pl) {
              const int p = 2 * k + pl;
              const uint64_t ad = q_desc + p * kSlotDesc;
              const uint64_t bd = k_desc + slot * kSlotDesc + pl * (kSlotDesc / 2);
              umma_ss_pair(s_tmem, ad, bd, idesc_qk, p != 0 ? 1u : 0u);
              umma_ss_pair(s_tmem, ad + 2, bd + 2, idesc_qk, 1u);
              umma_ss_pair(s_tmem, ad + 4, bd + 4, idesc_qk, 1u);
              umma_ss_pair(s_tmem, ad + 6, bd + 6, idesc_qk, 1u);
            }
            umma_commit_pair(bar(C::B_EMPTY + slot), kBoth);
            PA_TRACE_ONLY(tlog(3, tln, 4, round * NSLOT + slot);)
            advance();
          }
          if (!ok) break;
          umma_commit_pair(bar(C::B_SFULL + (j & 1)), kBoth);
        }
        if (j >= 1) {
          const int i = j - 1;
          PA_TRACE_ONLY(tlog(6, tln_w, 14, i);)
          PA_UNIT_ONLY(const long long c0 = clock64();)
          ok = wait_cluster(bar(C::B_PFULL + (i & 1)), (i >> 1) & 1);
          PA_UNIT_ONLY(w_p += clock64() - c0; w_sel = &w_v;)
          PA_TRACE_ONLY(tlog(3, tln, 5, i);)
          // Each half of the V tile (keys 0-63, then 64-127) is multiplied as soon as its slot
          // has landed, and its slot is released right after its four MMAs.
          const uint32_t p_tmem = tmem + kSCol0 + 128u * (i & 1) + kPColOff;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (ok) ok = wait_slot();
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 4 * h; ks < 4 * h + 4; ++ks) {
              const uint32_t off = v_offset_pair(16u * ks, 0, a.v_shift);
              umma_ts_pair(tmem + kOCol, p_tmem + ks * 8,
                           v_desc + slot * kSlotDesc + ((off & (kPanel - 1)) >> 4), idesc_pv,
                           (i > 0 || ks > 0) ? 1u : 0u);
            }
            umma_commit_pair(bar(C::B_EMPTY + slot), kBoth);
            advance();
          }
          if (!ok) break;
          PA_TRACE_ONLY(tlog(3, tln, 6, round * NSLOT + slot - 2);)
          umma_commit_pair(bar(C::B_PVDONE + (i & 1)), kBoth);
          PA_TRACE_ONLY(tlog(3, tln, 7, i);)
        }
      }
      PA_UNIT_ONLY(if (blockIdx.x < 8192) {
        g_pa_units[kUnitWords * blockIdx.x + 12] = (unsigned long long)w_k;
        g_pa_units[kUnitWords * blockIdx.x + 13] = (unsigned long long)w_v;
        g_pa_units[kUnitWords * blockIdx.x + 14] = (unsigned long long)w_p;
      })
      umma_commit_pair(bar(C::B_MMADONE), kBoth);
      drain_wait(bar(C::B_MMADONE), 0, abort_flag, tmo);
    }
    __syncwarp();
  } else {
    // ============================================================ rank 1, MMA warp
    // rank 0's last MMA has read this CTA's shared and tensor memory
    if (lane == 0) drain_wait(bar(C::B_MMADONE), 0, abort_flag, tmo);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  PA_UNIT_ONLY(if (threadIdx.x == 0 && blockIdx.x < 8192) {
    unsigned long long* u = g_pa_units + kUnitWords * blockIdx.x;
    u[0] = t_entry;
    u[1] = globaltimer_ns();
    u[2] = (uint64_t)n | ((uint64_t)smid_u32() << 32);
    u[3] = (uint64_t)c_entry;
    u[7] = (uint64_t)clock64();
  })
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
