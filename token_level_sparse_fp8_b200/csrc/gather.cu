// Gather-then-attend (the ablation the gather-free attention is measured against; JSSA README,
// "Highlights" and section 3: attending to the selected rows in place instead of first copying
// them; JSSA summary, section 3.3).
//
// Step 1 (this kernel): copy each (sequence, KV head)'s selected K and V rows, in index order,
// into contiguous staging buffers laid out like a paged cache of 16-token pages,
// [batch, budget_pad, h_kv, d] with budget_pad = budget rounded up to 16, so that step 2 is the
// dense paged decode over the staging buffers (sequence b = pages b * budget_pad / 16 ...,
// length count[b, 0]). Grid (row blocks of kRows index slots, batch * h_kv); each thread moves
// 16-byte chunks, all loads of a pass in flight before its stores.
#include "common.cuh"

namespace jssa {

namespace gather_detail {

constexpr int kThreads = 256;
constexpr int kRows = 64;  // index slots per CTA

struct GatherArgs {
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  int64_t page_stride, slot_stride, head_stride;
  const int32_t* block_table;
  int max_pages;
  const int32_t* idx;
  const int32_t* count;
  int h_kv, d, budget, budget_pad;
  int64_t num_pages;
  int page_size;
  uint16_t* k_out;
  uint16_t* v_out;
  int32_t* lens_out;
};

template <int D>
__global__ void __launch_bounds__(kThreads) gather_kernel(GatherArgs a) {
  constexpr int kChunks = D / 8;                 // 16-byte chunks per row
  constexpr int kRowsPerPass = kThreads / kChunks;
  const int pair = blockIdx.y;
  const int b = pair / a.h_kv, h = pair % a.h_kv;
  const int max_len = a.max_pages * a.page_size;
  int n = a.count[pair];
  n = n < 0 ? 0 : (n > a.budget ? a.budget : n);
  if (h == 0 && blockIdx.x == 0 && threadIdx.x == 0) a.lens_out[b] = n;
  const int j0 = blockIdx.x * kRows;
  const int row_in_pass = threadIdx.x / kChunks, c = threadIdx.x % kChunks;
  constexpr int kPasses = kRows / kRowsPerPass;
  uint4 kv[kPasses], vv[kPasses];
  int64_t dst[kPasses];
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    const int j = j0 + p * kRowsPerPass + row_in_pass;
    dst[p] = -1;
    kv[p] = vv[p] = make_uint4(0u, 0u, 0u, 0u);
    if (j >= n) continue;
    const int pos = a.idx[(int64_t)pair * a.budget + j];
    dst[p] = (((int64_t)b * a.budget_pad + j) * a.h_kv + h) * D + c * 8;
    if (pos < 0 || pos >= max_len) {
      if (c == 0) raise_flag(2u);
      continue;
    }
    const int pg = a.block_table[(int64_t)b * a.max_pages + pos / a.page_size];
    if (pg < 0 || (int64_t)pg >= a.num_pages) {
      if (c == 0) raise_flag(1u);
      continue;
    }
    const int64_t src = (int64_t)pg * a.page_stride + (int64_t)(pos % a.page_size) * a.slot_stride +
                        (int64_t)h * a.head_stride + c * 8;
    kv[p] = *reinterpret_cast<const uint4*>(a.k_cache + src);
    vv[p] = *reinterpret_cast<const uint4*>(a.v_cache + src);
  }
#pragma unroll
  for (int p = 0; p < kPasses; ++p) {
    if (dst[p] < 0) continue;
    *reinterpret_cast<uint4*>(a.k_out + dst[p]) = kv[p];
    *reinterpret_cast<uint4*>(a.v_out + dst[p]) = vv[p];
  }
}

}  // namespace gather_detail

cudaError_t launch_gather(const uint16_t* k_cache, const uint16_t* v_cache, int64_t page_stride,
                          int64_t slot_stride, int64_t head_stride, const int32_t* block_table,
                          int max_pages, const int32_t* idx, const int32_t* count, int batch,
                          int h_kv, int d, int budget, int64_t num_pages, int page_size,
                          uint16_t* k_out, uint16_t* v_out, int32_t* lens_out, cudaStream_t s) {
  using namespace gather_detail;
  if (batch * h_kv == 0) return cudaSuccess;
  GatherArgs a = {k_cache, v_cache, page_stride, slot_stride, head_stride, block_table, max_pages,
                  idx, count, h_kv, d, budget, (budget + 15) / 16 * 16, num_pages, page_size,
                  k_out, v_out, lens_out};
  dim3 grid((budget + kRows - 1) / kRows, batch * h_kv);
  if (d == 128) gather_kernel<128><<<grid, kThreads, 0, s>>>(a);
  else if (d == 256) gather_kernel<256><<<grid, kThreads, 0, s>>>(a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace jssa
