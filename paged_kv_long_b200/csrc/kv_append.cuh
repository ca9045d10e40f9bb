// kv_append.cuh — the step before prefill: write a chunk's new K and V rows into the paged pools
// through the page table (BaseRT issue #51, "Results": the chunk's K/V are published to pages,
// and prefill then reads every key, the chunk's own included, through the table). Included by
// pa_kernels.cu.
//
// Position p = H + i of chunk row i lives in page page_table[p / PS], slot p % PS. A pool slot
// [page][slot] holds all KV heads of one position contiguously (Hkv * D 16-bit values), so a
// row is row_vecs 16-byte pieces, contiguous on both sides. The K and V rows of all positions
// form one flat list of pieces per tensor (piece f = position f / row_vecs, piece f % row_vecs);
// warp w copies pieces 128w .. 128w + 127 of both tensors, four per lane and tensor, with all
// eight loads issued before the stores. At Hkv * D = 512 (c5) a warp moves two positions.
// Per-position warps, whose two pieces per lane and tensor gave four loads in flight and twice
// the blocks, measured 22.6 against 19.3 microseconds on c5's 32,768 rows. The work is
// HBM-bound (each byte read once and written once).

constexpr int kAppendBatch = 4;  // pieces per lane and tensor

__global__ void __launch_bounds__(256) kv_append_kernel(
    const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_pool,
    uint4* __restrict__ v_pool, const int32_t* __restrict__ page_table, int64_t num_pages,
    int64_t hist_len, int64_t rows, int page_size, int row_vecs) {
  const int lane = threadIdx.x & 31;
  const int64_t total = rows * row_vecs;
  const int64_t f0 = ((int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32) * 32 * kAppendBatch;
  uint4 kv[kAppendBatch], vv[kAppendBatch];
  int64_t dst[kAppendBatch];
#pragma unroll
  for (int u = 0; u < kAppendBatch; ++u) {
    const int64_t f = f0 + lane + 32 * u;
    dst[u] = -1;
    if (f < total) {
      const int64_t i = f / row_vecs;
      const int c = (int)(f - i * row_vecs);
      const int64_t pos = hist_len + i;
      const int32_t e = __ldg(page_table + pos / page_size);
      if (e < 0 || e >= num_pages) {  // the row is skipped, reported through the error word
        if (c == 0) atomicOr(&g_pa_error_flags, kFlagPage);
        continue;
      }
      dst[u] = ((int64_t)e * page_size + pos % page_size) * row_vecs + c;
      kv[u] = __ldg(k_new + f);
      vv[u] = __ldg(v_new + f);
    }
  }
#pragma unroll
  for (int u = 0; u < kAppendBatch; ++u) {
    if (dst[u] >= 0) {
      k_pool[dst[u]] = kv[u];
      v_pool[dst[u]] = vv[u];
    }
  }
}
