// decode_kernel.cuh — one decode step (one query token per sequence: pa_decode with device-side
// lengths, or a one-row batch with host-side lengths) with the operands of both products
// swapped. Included by pa_kernels.cu.
//
// A decode unit (sequence, KV head, split) has G <= 8 query rows, so a 128-row Q tile is almost
// all padding. Here the keys take the MMA's M side instead:
//   S^T = K Q^T:  A = the K tile (128 keys x D, K-major, as loaded), B = Q (16 rows: the G heads
//                 in one 8-row swizzle atom per 64-dim panel, repeated by a descriptor stride of
//                 0), D = 128 lanes (keys) x 16 columns (heads) of tensor memory;
//   O^T += V^T P^T: A = the V tile read MN-major (M = 128 dims, K = 16 keys per step), B = P^T
//                 (16 rows: heads, K = keys) written to shared memory by the softmax threads,
//                 D = 128 lanes (dims) x 16 columns per 128 dims.
// Tensor work per tile drops from 2 x 128 x 128 x D to 2 x 128 x 16 x D multiply-adds, and the
// accumulators take 64 columns of tensor memory instead of 512, so two CTAs share an SM: one
// CTA's set-up, first-tile latency and epilogue overlap the other's K/V stream. Each CTA keeps a
// ring of six 16 KB slots (K0, K1, V0, K2, V1, ... as in the single-CTA kernel).
//
// Softmax (warps 0-3, thread t = key t of the tile): per head, the tile's maximum is a warp
// reduction and a 4-warp exchange through shared memory (one named barrier per tile, which
// also carries a failed wait to every warp so that all leave the loop together); the running
// maximum is the same in every thread, the sums of the weights are per thread and added up
// once at the end. O^T is rescaled (a column per head, by the threads that own its lanes)
// only when some head's maximum grows by more than 2^8, as in the prefill kernels.

constexpr int kDecN = 16;                // N of both MMAs (heads 8..15 repeat 0..7)
constexpr int kDecSlots = 6;             // ring slots per CTA
constexpr uint32_t kDecTmemCols = 64;
constexpr uint32_t kDecSCol = 0;         // S^T buffers: columns [0, 16) and [16, 32)
constexpr uint32_t kDecOCol = 32;        // O^T: 16 columns per 128 dims
constexpr uint32_t kDecBarSoftmax = 1;   // named barrier of the 4 softmax warps

template <int D>
struct DecCfg {
  static constexpr int NP = D / 64;
  static constexpr int NSLOT = kDecSlots;
  static constexpr int Q_OFF = 0;                       // NP atoms of 8 rows x 128 B
  static constexpr int P_OFF = Q_OFF + NP * 1024;       // 2 buffers x 2 panels (64 keys) x 1 KB
  static constexpr int RING_OFF = P_OFF + 2 * 2 * 1024;
  static constexpr int BAR_OFF = RING_OFF + NSLOT * kPanel;
  static constexpr int B_FULL = 0, B_EMPTY = NSLOT, B_QFULL = 2 * NSLOT, B_SFULL = 2 * NSLOT + 1,
                       B_PFULL = 2 * NSLOT + 3, B_PVDONE = 2 * NSLOT + 5,
                       B_MMADONE = 2 * NSLOT + 7, N_BARS = 2 * NSLOT + 8;
  static constexpr int RED_OFF = BAR_OFF + 8 * N_BARS;  // [2][4 warps][8 heads] tile maxima
  static constexpr int SUM_OFF = RED_OFF + 2 * 4 * 8 * 4;  // [4 warps][8 heads] weight sums
  static constexpr int MISC_OFF = SUM_OFF + 4 * 8 * 4;
  static constexpr int SMEM = MISC_OFF + 16;
  static constexpr int LAUNCH_SMEM = SMEM + 1024;
  static constexpr int PANEL_LOG = (NP == 4) ? 9 : 8;
  static_assert(D == 128 || D == 256, "the swapped decode kernel takes head dim 128 or 256");
  static_assert(kDecCtasPerSm * (LAUNCH_SMEM + 1024) <= 233472, "two CTAs per SM");
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <bool BF16>
__device__ __forceinline__ uint16_t to16(float x) {
  if constexpr (BF16)
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
  else
    return __half_as_ushort(__float2half_rn(x));
}

// BAL: block b runs work item b of a balanced one-row batch (the item's sequence, KV head and
// key range; an uncut row block writes the output, a part of a cut one its partial and LSE in
// the item's workspace slot, merged by combine_blocks_kernel). Otherwise block b is decode unit
// b of pa_decode (device lengths, uniform splits).
template <int D, bool BF16, bool BAL>
__device__ __forceinline__ void decode_body(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                            const PrefillArgs& a_in, const ItemTable* items) {
  PrefillArgs a = a_in;
  using C = DecCfg<D>;
  constexpr int NP = C::NP, NSLOT = C::NSLOT, NH = D / 128;  // NH: 128-dim halves of O^T
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int g, s = 0, slot = kSlotUniform;
  int64_t kt0, kt1;
  if constexpr (BAL) {
    const PaItem it = items->item[blockIdx.x];
    const int32_t rb = batch_rebase<D>(a, *items, it.rb);  // one Q tile per sequence: g = rb
    int64_t qt;
    rb_coords(rb, a.q_tiles, a.Hkv, &qt, &g);
    kt0 = it.kt0;
    kt1 = it.kt1;
    slot = it.slot;
  } else {
    decode_unit<D>(a, reinterpret_cast<int32_t*>(smem + C::RING_OFF), &g, &s, &kt0, &kt1);
  }
  const int n = (int)(kt1 - kt0);
  if (n == 0) {
    empty_unit<D>(a, 0, g, s);
    return;
  }

  int32_t pre_row0 = a.oob_row, pre_row1 = a.oob_row;
  if (warp > kMmaWarp) {
    const bool report = warp == kMmaWarp + 1;
    pre_row0 = tile_page_row<true>(a, kt0, n, 0, lane, report);
    pre_row1 = tile_page_row<true>(a, kt0, n, 1, lane, report);
  }
  auto bar = [&](int i) -> uint32_t { return sb + C::BAR_OFF + 8u * (uint32_t)i; };
  auto slot_addr = [&](uint32_t r) -> uint32_t { return sb + C::RING_OFF + r * kPanel; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(bar(C::B_FULL + i), 1);
      mbar_init(bar(C::B_EMPTY + i), 1);
    }
    mbar_init(bar(C::B_QFULL), 1);
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
    tmem_alloc(smem_u32(tmem_slot), kDecTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;

  if (warp < 4) {
    // ============================================================ softmax + epilogue
    const int t = threadIdx.x;  // key t of each tile (S^T lane); dim t of each half (O^T lane)
    const int G = a.G;          // <= 8
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    if (warp == 0) {
      // Q rows 0..7 (heads g*G .. g*G+G-1, zeros past G), 128-byte swizzle, one atom per panel
      if (lane < 8) {
        const bool live = lane < G;
        const uint4* src =
            reinterpret_cast<const uint4*>(a.q + (int64_t)(g * G + (live ? lane : 0)) * D);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = live ? __ldg(src + p * 8 + c) : make_uint4(0u, 0u, 0u, 0u);
            st_shared_v4(sb + C::Q_OFF + p * 1024 + lane * 128 + ((c ^ lane) << 4), v.x, v.y,
                         v.z, v.w);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_QFULL));
    }
    float* red = reinterpret_cast<float*>(smem + C::RED_OFF);
    float* sums = reinterpret_cast<float*>(smem + C::SUM_OFF);
    float m_run[8], l_part[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      m_run[h] = -INFINITY;
      l_part[h] = 0.f;
    }
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int sbuf = j & 1;
      const int64_t key0 = (kt0 + j) * kTileKeys;
      const bool live = key0 + t < a.total_keys;
      float sv[8];
      if (ok) ok = warp_wait(bar(C::B_SFULL + sbuf), (j >> 1) & 1, abort_flag, tmo);
      if (ok) {
        tc_fence_after();
        tmem_ld8(t_lane + kDecSCol + 16u * sbuf, sv);
        tmem_wait_ld();
      }
      float mx[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) mx[h] = warp_max(ok && live ? sv[h] : -INFINITY);
      if (lane == 0) {
        float* r = red + sbuf * 32 + warp * 8;
        *reinterpret_cast<float4*>(r) = make_float4(mx[0], mx[1], mx[2], mx[3]);
        *reinterpret_cast<float4*>(r + 4) = make_float4(mx[4], mx[5], mx[6], mx[7]);
      }
      if (named_bar_or(kDecBarSoftmax, 128, !ok)) {
        ok = false;
        break;
      }
      // The tile's maximum per head over the four warps (the same in every thread). red[sbuf]
      // is written again two tiles on, after every warp has passed the next tile's barrier.
      float m_new[8];
      bool need[8], any = false;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float* r = red + sbuf * 32 + h;
        const float tm = fmaxf(fmaxf(r[0], r[8]), fmaxf(r[16], r[24]));
        m_new[h] = fmaxf(m_run[h], tm * a.scale_log2);
        need[h] = m_new[h] > m_run[h] + kRescaleLog2;
        any |= need[h];
      }
      if (j == 0) {
#pragma unroll
        for (int h = 0; h < 8; ++h)
          if (need[h]) m_run[h] = m_new[h];
      } else if (any) {
        // O^T must not change under a running MMA: wait for PV of the previous tile.
        ok = warp_wait(bar(C::B_PVDONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag, tmo);
        if (ok) {
          tc_fence_after();
          float f[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            f[h] = need[h] ? ex2(m_run[h] - m_new[h]) : 1.0f;
            l_part[h] *= f[h];
            if (need[h]) m_run[h] = m_new[h];
          }
#pragma unroll
          for (int hf = 0; hf < NH; ++hf) {
            float o[8];
            tmem_ld8(t_lane + kDecOCol + 16u * hf, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < 8; ++h) o[h] *= f[h];
            tmem_st8(t_lane + kDecOCol + 16u * hf, o);
          }
          tmem_wait_st();
        }
      }
      float p[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float mu = m_run[h] == -INFINITY ? 0.f : m_run[h];
        p[h] = ok && live ? ex2(fmaf(sv[h], a.scale_log2, -mu)) : 0.f;
        l_part[h] += p[h];
      }
      // P(j) goes to buffer j % 2 once PV(j-2), its last reader, is done. PV of tile i
      // completes phase i/2 of pv_done[i % 2]; as in the prefill kernels no phase is skipped.
      if (ok && j >= 2)
        ok = warp_wait(bar(C::B_PVDONE + sbuf), ((j - 2) >> 1) & 1, abort_flag, tmo);
      if (ok && key0 + kTileKeys > a.total_keys) {
        // The tail tile: V rows of keys past the sequence (in its last page) hold arbitrary
        // bits and P is 0 there, but 0 * NaN is NaN inside the MMA, so those rows are zeroed.
        // Once PV(j-1) is done, every earlier fill of V(j)'s slots has landed (the tail tile
        // is the unit's last), so the parity waits below see V(j)'s own fills.
        if (j >= 1)
          ok = warp_wait(bar(C::B_PVDONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag, tmo);
        const uint32_t seq0 = v_item(j, n) * NP;
        for (int q = 0; q < NP && ok; ++q)
          ok = warp_wait(bar(C::B_FULL + (seq0 + q) % NSLOT), ((seq0 + q) / NSLOT) & 1,
                         abort_flag, tmo);
        if (ok && !live) {
#pragma unroll
          for (int q = 0; q < NP; ++q) {
            const uint32_t off = v_offset<NP, C::PANEL_LOG>((uint32_t)t, q, a.v_shift);
            const uint32_t ra = slot_addr((seq0 + (off >> 14)) % NSLOT) + (off & (kPanel - 1));
#pragma unroll
            for (int c = 0; c < 8; ++c) st_shared_v4(ra + c * 16, 0u, 0u, 0u, 0u);
          }
        }
      }
      if (ok) {
        // P^T[h][t]: row h of the atom of keys 64*(t/64) .., 16-byte chunk (t % 64) / 8 ^ h
        const uint32_t pb = sb + C::P_OFF + (uint32_t)sbuf * 2048u + (uint32_t)(t >> 6) * 1024u;
        const uint32_t chunk = (uint32_t)((t & 63) >> 3), sub = (uint32_t)(t & 7) * 2u;
#pragma unroll
        for (int h = 0; h < 8; ++h)
          st_shared_u16(pb + h * 128u + ((chunk ^ (uint32_t)h) << 4) + sub, to16<BF16>(p[h]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(bar(C::B_PFULL + sbuf));
    }

    if (ok && n >= 2)
      ok = warp_wait(bar(C::B_PVDONE + ((n - 2) & 1)), ((n - 2) >> 1) & 1, abort_flag, tmo);
    if (ok) ok = warp_wait(bar(C::B_PVDONE + ((n - 1) & 1)), ((n - 1) >> 1) & 1, abort_flag, tmo);
    float ls[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) ls[h] = warp_sum(l_part[h]);
    if (lane == 0) {
      *reinterpret_cast<float4*>(sums + warp * 8) = make_float4(ls[0], ls[1], ls[2], ls[3]);
      *reinterpret_cast<float4*>(sums + warp * 8 + 4) = make_float4(ls[4], ls[5], ls[6], ls[7]);
    }
    if (!named_bar_or(kDecBarSoftmax, 128, !ok)) {
      tc_fence_after();
      float inv_l[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        ls[h] = (sums[h] + sums[8 + h]) + (sums[16 + h] + sums[24 + h]);
        inv_l[h] = ls[h] > 0.f ? 1.f / ls[h] : 0.f;
      }
      // Destination rows of heads g*G + h: the output, a uniform split's partial, or the packed
      // rows h of a balanced item's workspace slot.
      bool partial;
      int64_t row0;
      if (slot >= 0) {
        partial = true;
        row0 = (int64_t)slot * a.rows_per_block;
      } else {
        partial = slot == kSlotUniform && a.splits > 1;
        row0 = partial ? (int64_t)s * a.ws_split_rows + g * G : (int64_t)g * G;
      }
      float* base = partial ? a.ws_o : a.out;
#pragma unroll
      for (int hf = 0; hf < NH; ++hf) {
        float o[8];
        tmem_ld8(t_lane + kDecOCol + 16u * hf, o);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 8; ++h)
          if (h < G) base[(row0 + h) * D + 128 * hf + t] = o[h] * inv_l[h];
      }
      if (partial) {
#pragma unroll
        for (int h = 0; h < 8; ++h)
          if (t == h && h < G)
            a.ws_lse[row0 + h] = ls[h] > 0.f ? m_run[h] + log2f(ls[h]) : -INFINITY;
      }
    }
  } else if (warp > kMmaWarp) {
    // ============================================================ TMA issuers (three warps)
    kv_copy_role<NP, NSLOT, C::PANEL_LOG, true>(a, &tm_k, &tm_v, g, kt0, n, warp - kMmaWarp - 1,
                                                sb + C::RING_OFF, bar(C::B_FULL),
                                                bar(C::B_EMPTY), pre_row0, pre_row1, abort_flag,
                                                tmo);
  } else {
    // ============================================================ MMA issuer (one lane)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_f16(128, kDecN, BF16, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_f16(128, kDecN, BF16, false, true);
      constexpr uint32_t kSlotDesc = kPanel >> 4;
      const uint64_t q_desc = smem_desc_sw128(sb + C::Q_OFF, 16, 0);
      const uint64_t p_desc = smem_desc_sw128(sb + C::P_OFF, 16, 0);
      const uint64_t k_desc = smem_desc_sw128(sb + C::RING_OFF, 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(sb + C::RING_OFF, (uint32_t)a.v_rows * 128u, 1024);
      uint32_t slot = 0, round = 0;
      bool ok = thread_wait(bar(C::B_QFULL), 0, abort_flag, tmo);
      tc_fence_after();
      for (int j = 0; j <= n && ok; ++j) {
        if (j < n) {
          // S^T_j is written over S^T_{j-2}, which the softmax read before it released P_{j-2}
          // (the PV MMA that read P_{j-2} was issued before this one).
          const uint32_t s_tmem = tmem + kDecSCol + 16u * (j & 1);
#pragma unroll
          for (int p = 0; p < NP; ++p) {
            ok = thread_wait(bar(C::B_FULL + slot), round & 1, abort_flag, tmo);
            if (!ok) break;
            tc_fence_after();
            const uint64_t ad = k_desc + slot * kSlotDesc, bd = q_desc + p * (1024 >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_ss(s_tmem, ad + 2 * kk, bd + 2 * kk, idesc_qk, (p | kk) != 0 ? 1u : 0u);
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
          const uint32_t vslot0 = slot;
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
#pragma unroll
          for (int ks = 0; ks < kTileKeys / 16; ++ks) {
            const uint64_t bd = p_desc + (uint32_t)(i & 1) * (2048 >> 4) + (ks >> 2) * (1024 >> 4) +
                                (ks & 3) * 2;
#pragma unroll
            for (int hf = 0; hf < NH; ++hf) {
              const uint32_t off = v_offset<NP, C::PANEL_LOG>(16u * ks, 2u * hf, a.v_shift);
              uint32_t vs = vslot0 + (off >> 14);
              if (vs >= (uint32_t)NSLOT) vs -= NSLOT;
              umma_ss(tmem + kDecOCol + 16u * hf,
                      v_desc + vs * kSlotDesc + ((off & (kPanel - 1)) >> 4), bd, idesc_pv,
                      (i > 0 || ks > 0) ? 1u : 0u);
            }
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
    tmem_dealloc(tmem, kDecTmemCols);
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, kDecCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const PrefillArgs a) {
  decode_body<D, BF16, false>(tm_k, tm_v, a, nullptr);
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads, kDecCtasPerSm)
    decode_batch_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a,
                        const __grid_constant__ ItemTable items) {
  decode_body<D, BF16, true>(tm_k, tm_v, a, &items);
}
