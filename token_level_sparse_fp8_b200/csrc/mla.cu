// Multi-head latent attention (MLA) over selected positions, in the absorbed form (JSSA summary,
// section 3.3, and JSSA README, paper-to-code map and section 4 notes: the MLA path keeps one
// latent row per token, 512 latent + 64 rotary dimensions, and attends to the selected rows in
// place):
//
//   out[b, i, :] = sum_j softmax_j(scale * q[b, i] . kv[j]) kv[j, 0:512]   (j in the index set)
//
// with q the absorbed queries (576 = 512 + 64 per head), kv the paged latent cache (576 bf16 per
// token, one "KV head") and the index set of score_topk run with h_kv = 1 on the latent scoring
// cache.
//
// Grid (h_q / 16, splits, batch): a CTA owns 16 query heads of one sequence and one contiguous
// slice of its index set; the head blocks of one slice are neighbours in launch order, so the
// rows they all read come from L2 after the first. Its 4 warps share every 16-token tile of latent rows (a CTA-wide ring
// of kStages shared-memory stages filled by 16-byte cp.async, chunk c of a row at
// (c & ~7) | ((c ^ row) & 7) so that ldmatrix reads are conflict-free). The scores S = Q K^T of
// the 16 heads x 16 tokens are computed on the tensor cores (mma.sync m16n8k16 bf16, fp32
// accumulate; the 16 heads are the M rows) with the 576 dimensions split over the 4 warps (9
// k-blocks each) and the partial sums added through shared memory; every warp then keeps the
// same online softmax and adds P V into its quarter (128 dims) of the output (P split into bf16
// high and low parts). Splits
// of one (sequence, head block) merge through fp32 partials and a ticket, as the GQA attention.
#include "common.cuh"

namespace jssa {

namespace mla_detail {

constexpr int kDK = 576;             // latent + rotary dimensions of a key row
constexpr int kDV = 512;             // latent dimensions (the value row)
constexpr int kHeads = 16;           // query heads per CTA (the MMA's M rows)
constexpr int kWarps = 4;            // each owns kDV / kWarps output dimensions
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 16;            // tokens per tile
constexpr int kStages = 3;
constexpr int kRowBytes = kDK * 2;   // 1152
constexpr int kChunks = kRowBytes / 16;  // 72
constexpr int kTileBytes = kTile * kRowBytes;
constexpr int kQBytes = kHeads * kRowBytes;
constexpr int kMaxChunk = 1024;      // positions per CTA
constexpr int kSmem = kQBytes + kStages * kTileBytes;
constexpr int kDimsPerWarp = kDV / kWarps;  // 128
constexpr int kMaxMergeSplits = kStages * kTileBytes / (kHeads * 3 * 4);  // 288

struct Args {
  const uint16_t* q;
  const uint16_t* kv;
  int64_t page_stride, slot_stride;
  const int32_t* block_table;
  int max_pages;
  const int32_t* idx;
  const int32_t* count;
  int batch, h_q, budget;
  int64_t num_pages;
  int page_size;
  float scale;
  uint16_t* out;
  void* ws;
};

__device__ __forceinline__ uint32_t swz(int row, int c) {
  return (uint32_t)(row * kRowBytes + (((c & ~7) | ((c ^ row) & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads, 2) mla_kernel(Args a, int chunk, int splits) {
  extern __shared__ __align__(128) uint8_t mla_smem[];
  __shared__ int64_t s_off[kMaxChunk];
  __shared__ float s_part[kWarps][32][8];  // each warp's partial S, in fragment order
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int hb = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int n_hb = gridDim.x;
  const int max_len = a.max_pages * a.page_size;
  const uint32_t s_q = smem_u32(mla_smem);
  const uint32_t ring = s_q + kQBytes;

  // the 16 heads' absorbed queries (inputs of the step, complete before it) -> shared memory
  {
    const uint16_t* qb = a.q + ((int64_t)b * a.h_q + (int64_t)hb * kHeads) * kDK;
    for (int i = tid; i < kHeads * kChunks; i += kThreads) {
      const int row = i / kChunks, c = i % kChunks;
      cp_async16(s_q + swz(row, c), qb + (int64_t)row * kDK + c * 8, 16);
    }
    cp_async_commit();
  }
  pdl_wait();  // index sets come from the preceding score + top-B kernel
  int n_total = a.count[b];
  n_total = n_total < 0 ? 0 : (n_total > a.budget ? a.budget : n_total);
  const int j_begin = split * chunk;
  const int n_mine = max(0, min(chunk, n_total - j_begin));
  {
    constexpr int kPer = kMaxChunk / kThreads;
    const int32_t* bt = a.block_table + (int64_t)b * a.max_pages;
    int pos[kPer], pg[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int j = tid + u * kThreads;
      pos[u] = j < n_mine ? a.idx[(int64_t)b * a.budget + j_begin + j] : -1;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const bool in = pos[u] >= 0 && pos[u] < max_len;
      pg[u] = in ? bt[pos[u] / a.page_size] : -1;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int j = tid + u * kThreads;
      if (j >= n_mine) continue;
      int64_t off = -1;
      if (pos[u] < 0 || pos[u] >= max_len) raise_flag(2u);
      else if (pg[u] < 0 || (int64_t)pg[u] >= a.num_pages) raise_flag(1u);
      else off = (int64_t)pg[u] * a.page_stride + (int64_t)(pos[u] % a.page_size) * a.slot_stride;
      s_off[j] = off;
    }
  }
  __syncthreads();
  pdl_trigger();

  const int n_tiles = (n_mine + kTile - 1) / kTile;
  // copies of a tile: 8 threads per row, thread q of a row takes chunks q, q + 8, ..., q + 64 (a
  // warp instruction covers 128 contiguous bytes of each of its 4 rows); the swizzle only flips
  // the low 3 bits of the chunk index, so a thread's destinations are 128 bytes apart
  static_assert(kThreads == kTile * 8 && kChunks % 8 == 0, "copy split");
  const int cp_row = tid >> 3, cp_q = tid & 7;
  const uint32_t cp_dst = (uint32_t)(cp_row * kRowBytes + ((cp_q ^ (cp_row & 7)) << 4));
  auto issue = [&](int tl, int st) {
    const int j = tl * kTile + cp_row;
    const int64_t off = j < n_mine ? s_off[j] : -1;
    const uint16_t* src = a.kv + (off >= 0 ? off : 0) + cp_q * 8;
    const uint32_t dst = ring + st * kTileBytes + cp_dst;
#pragma unroll
    for (int k = 0; k < kChunks / 8; ++k) cp_async16(dst + 128 * k, src + 64 * k, off >= 0 ? 16 : 0);
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < n_tiles) issue(i, i);
    cp_async_commit();
  }

  const float scale_log2 = a.scale * 1.4426950408889634f;
  float o[kDimsPerWarp / 8][4];
#pragma unroll
  for (int n = 0; n < kDimsPerWarp / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // rows g, g + 8
  // ldmatrix lane roles
  const int mat = lane >> 3, mr = lane & 7;
  const int qa_row = mr + (mat & 1) * 8, qa_half = mat >> 1;   // Q (A): heads 0-7 / 8-15, k lo / hi
  const int kb_row = mr + (mat >> 1) * 8, kb_half = mat & 1;   // K (B): tokens 0-7 / 8-15, k lo / hi
  const int vb_row = mr + (mat & 1) * 8, vb_next = mat >> 1;   // V (B, trans): tokens lo / hi, n-tile

  for (int i = 0; i < n_tiles; ++i) {
    if (i + kStages - 1 < n_tiles) issue(i + kStages - 1, (i + kStages - 1) % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncthreads();
    const uint32_t st = ring + (i % kStages) * kTileBytes;

    // S (16 heads x 16 tokens) = Q K^T over the 576 dimensions: this warp's 9 k-blocks, then
    // the four partial sums through shared memory (the same fragment order in every warp)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    constexpr int kKB = kDK / 16 / kWarps;  // 9
#pragma unroll
    for (int u = 0; u < kKB; ++u) {
      const int kb = warp * kKB + u;
      uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
      ldsm_x4(s_q + swz(qa_row, 2 * kb + qa_half), a0, a1, a2, a3);
      ldsm_x4(st + swz(kb_row, 2 * kb + kb_half), b0, b1, b2, b3);
      mma_bf16(s0, a0, a1, a2, a3, b0, b1);
      mma_bf16(s1, a0, a1, a2, a3, b2, b3);
    }
    *reinterpret_cast<float4*>(&s_part[warp][lane][0]) = make_float4(s0[0], s0[1], s0[2], s0[3]);
    *reinterpret_cast<float4*>(&s_part[warp][lane][4]) = make_float4(s1[0], s1[1], s1[2], s1[3]);
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s0[e] = s_part[0][lane][e] + s_part[1][lane][e] + s_part[2][lane][e] + s_part[3][lane][e];
      s1[e] = s_part[0][lane][4 + e] + s_part[1][lane][4 + e] + s_part[2][lane][4 + e] +
              s_part[3][lane][4 + e];
    }
    // rows g (s[0], s[1]) and g + 8 (s[2], s[3]); columns: tokens 2t, 2t + 1 (+ 8 in s1)
    const int j0 = i * kTile;
    const bool v00 = j0 + 2 * t < n_mine && s_off[j0 + 2 * t] >= 0;
    const bool v01 = j0 + 2 * t + 1 < n_mine && s_off[j0 + 2 * t + 1] >= 0;
    const bool v10 = j0 + 8 + 2 * t < n_mine && s_off[j0 + 8 + 2 * t] >= 0;
    const bool v11 = j0 + 9 + 2 * t < n_mine && s_off[j0 + 9 + 2 * t] >= 0;
    float x[8];
    x[0] = v00 ? s0[0] * scale_log2 : -INFINITY;  // row g
    x[1] = v01 ? s0[1] * scale_log2 : -INFINITY;
    x[2] = v10 ? s1[0] * scale_log2 : -INFINITY;
    x[3] = v11 ? s1[1] * scale_log2 : -INFINITY;
    x[4] = v00 ? s0[2] * scale_log2 : -INFINITY;  // row g + 8
    x[5] = v01 ? s0[3] * scale_log2 : -INFINITY;
    x[6] = v10 ? s1[2] * scale_log2 : -INFINITY;
    x[7] = v11 ? s1[3] * scale_log2 : -INFINITY;
    float mx0 = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    float mx1 = fmaxf(fmaxf(x[4], x[5]), fmaxf(x[6], x[7]));
#pragma unroll
    for (int sh = 1; sh < 4; sh <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, sh));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, sh));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float corr0 = fast_exp2(m_run[0] - mu0), corr1 = fast_exp2(m_run[1] - mu1);
    float p[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = fast_exp2(x[e] - mu0);
      p[4 + e] = fast_exp2(x[4 + e] - mu1);
    }
    l_run[0] = l_run[0] * corr0 + (p[0] + p[1] + p[2] + p[3]);
    l_run[1] = l_run[1] * corr1 + (p[4] + p[5] + p[6] + p[7]);
    m_run[0] = mn0;
    m_run[1] = mn1;
#pragma unroll
    for (int n = 0; n < kDimsPerWarp / 8; ++n) {
      o[n][0] *= corr0;
      o[n][1] *= corr0;
      o[n][2] *= corr1;
      o[n][3] *= corr1;
    }
    // P as the A operand (16 heads x 16 tokens), high and low bf16 parts
    const uint32_t h0 = pack_bf16x2(p[0], p[1]), h1 = pack_bf16x2(p[4], p[5]);
    const uint32_t h2 = pack_bf16x2(p[2], p[3]), h3 = pack_bf16x2(p[6], p[7]);
    const uint32_t l0 = pack_bf16x2(p[0] - bf16_lo(h0), p[1] - bf16_hi(h0));
    const uint32_t l1 = pack_bf16x2(p[4] - bf16_lo(h1), p[5] - bf16_hi(h1));
    const uint32_t l2 = pack_bf16x2(p[2] - bf16_lo(h2), p[3] - bf16_hi(h2));
    const uint32_t l3 = pack_bf16x2(p[6] - bf16_lo(h3), p[7] - bf16_hi(h3));
    // O (16 heads x this warp's 128 dims) += P V
#pragma unroll
    for (int n = 0; n < kDimsPerWarp / 8; n += 2) {
      const int c = (warp * kDimsPerWarp + n * 8) / 8 + vb_next;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(st + swz(vb_row, c), b0, b1, b2, b3);
      mma_bf16(o[n], h0, h1, h2, h3, b0, b1);
      mma_bf16(o[n], l0, l1, l2, l3, b0, b1);
      mma_bf16(o[n + 1], h0, h1, h2, h3, b2, b3);
      mma_bf16(o[n + 1], l0, l1, l2, l3, b2, b3);
    }
    __syncthreads();  // the stage is refilled by the next iteration's copies
  }
  cp_async_wait<0>();
#pragma unroll
  for (int sh = 1; sh < 4; sh <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], sh);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], sh);
  }

  const int head0 = hb * kHeads;
  const int64_t out_row0 = (int64_t)b * a.h_q + head0;
  if (splits == 1) {
#pragma unroll
    for (int n = 0; n < kDimsPerWarp / 8; ++n) {
      const int d0 = warp * kDimsPerWarp + n * 8 + 2 * t;
      const float i0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f, i1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
      *reinterpret_cast<uint32_t*>(a.out + (out_row0 + g) * kDV + d0) = pack_bf16x2(o[n][0] * i0, o[n][1] * i0);
      *reinterpret_cast<uint32_t*>(a.out + (out_row0 + g + 8) * kDV + d0) = pack_bf16x2(o[n][2] * i1, o[n][3] * i1);
    }
    return;
  }
  // partials [batch][head block][split][16 heads][2 + 512] (m in log2 units, l, o) and tickets
  const int64_t n_blocks = (int64_t)a.batch * n_hb;
  int* tickets = reinterpret_cast<int*>(a.ws);
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.ws) + ((n_blocks * 4 + 255) / 256) * 256);
  const int64_t blk = (int64_t)b * n_hb + hb;
  float* pb = part + (blk * splits + split) * kHeads * (kDV + 2);
  if (warp == 0 && t == 0) {
    __stcg(pb + g * (kDV + 2), m_run[0]);
    __stcg(pb + g * (kDV + 2) + 1, l_run[0]);
    __stcg(pb + (g + 8) * (kDV + 2), m_run[1]);
    __stcg(pb + (g + 8) * (kDV + 2) + 1, l_run[1]);
  }
#pragma unroll
  for (int n = 0; n < kDimsPerWarp / 8; ++n) {
    const int d0 = warp * kDimsPerWarp + n * 8 + 2 * t;
    __stcg(pb + g * (kDV + 2) + 2 + d0, o[n][0]);
    __stcg(pb + g * (kDV + 2) + 3 + d0, o[n][1]);
    __stcg(pb + (g + 8) * (kDV + 2) + 2 + d0, o[n][2]);
    __stcg(pb + (g + 8) * (kDV + 2) + 3 + d0, o[n][3]);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&tickets[blk], 1) == splits - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge: weights w = 2^(m - M) / L per (split, head) in shared memory (the ring is free), then
  // one weighted sum of independent loads per output element
  const float* p0 = part + blk * splits * kHeads * (kDV + 2);
  const int64_t step = (int64_t)kHeads * (kDV + 2);
  float* s_pm = reinterpret_cast<float*>(mla_smem + kQBytes);
  float* s_pl = s_pm + splits * kHeads;
  float* s_w = s_pl + splits * kHeads;
  for (int i = tid; i < splits * kHeads; i += kThreads) {
    const int sp = i / kHeads, row = i % kHeads;
    s_pm[i] = __ldcg(p0 + sp * step + (int64_t)row * (kDV + 2));
    s_pl[i] = __ldcg(p0 + sp * step + (int64_t)row * (kDV + 2) + 1);
  }
  __syncthreads();
  if (tid < kHeads) {
    float mm = -INFINITY;
    for (int sp = 0; sp < splits; ++sp) mm = fmaxf(mm, s_pm[sp * kHeads + tid]);
    float l = 0.f;
    if (mm != -INFINITY)
      for (int sp = 0; sp < splits; ++sp) l += fast_exp2(s_pm[sp * kHeads + tid] - mm) * s_pl[sp * kHeads + tid];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int sp = 0; sp < splits; ++sp)
      s_w[sp * kHeads + tid] = mm != -INFINITY ? fast_exp2(s_pm[sp * kHeads + tid] - mm) * inv : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < kHeads * kDV; e += kThreads) {
    const int row = e / kDV, dim = e % kDV;
    const float* pp = p0 + (int64_t)row * (kDV + 2) + 2 + dim;
    float acc = 0.f;
#pragma unroll 8
    for (int sp = 0; sp < splits; ++sp) acc += s_w[sp * kHeads + row] * __ldcg(pp + sp * step);
    a.out[(out_row0 + row) * kDV + dim] = f_to_bf16(acc);
  }
  if (tid == 0) tickets[blk] = 0;
}

}  // namespace mla_detail

MlaPlan plan_mla(int batch, int h_q, int budget) {
  using namespace mla_detail;
  MlaPlan p;
  const int blocks = batch * (h_q / kHeads);
  const int unit = 4 * kTile;  // at least 4 tiles per CTA
  int splits = (2 * num_sms()) / (blocks > 0 ? blocks : 1);
  const int max_splits = (budget + unit - 1) / unit;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int chunk = (budget + splits - 1) / splits;
  chunk = (chunk + unit - 1) / unit * unit;
  const int min_chunk = (budget + kMaxMergeSplits - 1) / kMaxMergeSplits;  // the merge buffer
  if (chunk < min_chunk) chunk = (min_chunk + unit - 1) / unit * unit;
  if (chunk > kMaxChunk) chunk = kMaxChunk;
  splits = (budget + chunk - 1) / chunk;
  p.splits = splits;
  p.chunk = chunk;
  p.ws_bytes = splits > 1 ? (((size_t)blocks * 4 + 255) / 256) * 256 +
                                (size_t)blocks * splits * kHeads * (kDV + 2) * sizeof(float)
                          : 0;
  return p;
}

cudaError_t launch_mla(const uint16_t* q, const uint16_t* kv, int64_t page_stride,
                       int64_t slot_stride, const int32_t* block_table, int max_pages,
                       const int32_t* idx, const int32_t* count, int batch, int h_q, int budget,
                       int64_t num_pages, int page_size, float scale, uint16_t* out, void* ws,
                       const MlaPlan& plan, bool pdl, cudaStream_t s) {
  using namespace mla_detail;
  if (batch == 0) return cudaSuccess;
  static_assert(kSmem >= kStages * kTileBytes, "merge buffer");
  cudaError_t e = configure_kernel((const void*)mla_kernel, kSmem, false);
  if (e != cudaSuccess) return e;
  Args a = {q, kv, page_stride, slot_stride, block_table, max_pages, idx, count, batch, h_q,
            budget, num_pages, page_size, scale, out, ws};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h_q / kHeads, plan.splits, batch);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, mla_kernel, a, plan.chunk, plan.splits);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace jssa
