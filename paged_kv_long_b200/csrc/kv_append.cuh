// kv_append.cuh — the step before prefill: write a chunk's new K and V rows into the paged pools
// through the page table (BaseRT issue #51, "Results": the chunk's K/V are published to pages,
// and prefill then reads every key, the chunk's own included, through the table). Included by
// pa_kernels.cu.
//
// Position p = H + i of chunk row i lives in page page_table[p / PS], slot p % PS. A pool slot
// [page][slot] holds all KV heads of one position contiguously (Hkv * D 16-bit values), so a
// row is one contiguous copy. One warp copies one position: its K row and its V row (the same
// page slot, one page-table read), in 16-byte pieces, with every load of a batch of up to four
// pieces per lane and tensor issued before its stores (up to eight loads in flight per lane).
// The work is HBM-bound (each byte read once and written once).

__global__ void __launch_bounds__(256) kv_append_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_pool,
    uint4* __restrict__ v_pool, const int32_t* __restrict__ page_table, int64_t num_pages,
    int64_t hist_len, int64_t rows, int page_size, int row_vecs) {
  const int64_t i = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (i >= rows) return;
  const int lane = threadIdx.x & 31;
  const int64_t pos = hist_len + i;
  const int32_t e = __ldg(page_table + pos / page_size);
  if (e < 0 || e >= num_pages) {  // skipped, reported through the device error word
    if (lane == 0) atomicOr(&g_pa_error_flags, kFlagPage);
    return;
  }
  const uint4* ks = k_new + i * row_vecs;
  const uint4* vs = v_new + i * row_vecs;
  const int64_t slot = ((int64_t)e * page_size + pos % page_size) * row_vecs;
  uint4* kd = k_pool + slot;
  uint4* vd = v_pool + slot;
  constexpr int kBatch = 4;
  for (int c0 = 0; c0 < row_vecs; c0 += 32 * kBatch) {
    uint4 kv[kBatch], vv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int c = c0 + lane + 32 * u;
      if (c < row_vecs) {
        kv[u] = __ldg(ks + c);
        vv[u] = __ldg(vs + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int c = c0 + lane + 32 * u;
      if (c < row_vecs) {
        kd[c] = kv[u];
        vd[c] = vv[u];
      }
    }
  }
}
