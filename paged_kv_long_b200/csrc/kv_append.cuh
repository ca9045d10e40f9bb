// kv_append.cuh — the step before prefill: write a chunk's new K and V rows into the paged pools
// through the page table (BaseRT issue #51, "Results": the chunk's K/V are published to pages,
// and prefill then reads every key, the chunk's own included, through the table). Included by
// pa_kernels.cu.
//
// Position p = H + i of chunk row i lives in page page_table[p / PS], slot p % PS. A pool slot
// [page][slot] holds all KV heads of one position contiguously (Hkv * D 16-bit values), so a
// row is one contiguous copy. One warp copies one row of K or of V in 16-byte pieces; the work
// is HBM-bound (each byte read once and written once).

__global__ void __launch_bounds__(256) kv_append_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_pool,
    uint4* __restrict__ v_pool, const int32_t* __restrict__ page_table, int64_t num_pages,
    int64_t hist_len, int64_t rows, int page_size, int row_vecs) {
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (w >= 2 * rows) return;
  const int lane = threadIdx.x & 31;
  const int64_t i = w >> 1;
  const bool is_v = (w & 1) != 0;
  const int64_t pos = hist_len + i;
  const int32_t e = __ldg(page_table + pos / page_size);
  if (e < 0 || e >= num_pages) {  // skipped, reported through the device error word
    if (lane == 0) atomicOr(&g_pa_error_flags, kFlagPage);
    return;
  }
  const uint4* src = (is_v ? v_new : k_new) + i * row_vecs;
  uint4* dst = (is_v ? v_pool : k_pool) + ((int64_t)e * page_size + pos % page_size) * row_vecs;
  for (int c = lane; c < row_vecs; c += 32) dst[c] = __ldg(src + c);
}
