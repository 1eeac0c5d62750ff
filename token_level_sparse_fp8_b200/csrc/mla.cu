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
// On the 5th-generation tensor cores, with every operand that is reused held in tensor memory.
// Grid (head blocks x 4, splits, batch): a CTA owns 128 query heads of one sequence (the M = 128
// rows of every MMA; a smaller h_q pads the block with zero queries), one quarter (128 of the
// 512) of the value dimensions and one contiguous slice of the index set. Tensor memory (512
// columns x 128 lanes, lane = head):
//   columns   0-287  Q, the A operand of S = Q K^T (576 bf16 per row, written once)
//   columns 288-351  S (64 tokens, fp32), then in place P = softmax weights as two bf16 parts
//                    (high 288-319, low 320-351: P V is two MMAs and the weights keep ~16 bits)
//   columns 384-511  O, this CTA's 128 value dimensions (fp32 accumulator)
// Latent rows arrive by 16-byte cp.async, 64 tokens per tile, in a 3-stage ring (tile i + 1 is
// copied into the stage of tile i - 2 while P V of tile i - 1 runs). A tile is kept
// as 9 column blocks of 64 dimensions (128 bytes per token, 128-byte swizzle), the layout that
// serves both as the K-major B operand of S (N = 64 tokens) and as the MN-major B operand of P V
// (N = 128 value dimensions, K = 64 tokens), so each row is read from L2 once per CTA. One
// thread issues the MMAs; 8 warps, two per 32 tensor-memory lanes (heads), each taking half of a
// tile's tokens, read S, keep the online softmax with a lazy rescale (O is rescaled through
// tensor memory only when a row's maximum grows by more than 2^8; the two halves exchange the
// row maximum through shared memory) and write P back. Every wait on the tensor cores is bounded
// (a timeout raises JSSA_DEVERR_TIMEOUT and the CTA still releases its tensor memory). Splits of
// one (sequence, head block, quarter) merge through fp32 partials and a ticket.
#include "common.cuh"
#include "tcgen05.cuh"

namespace jssa {

namespace mla_detail {

constexpr int kDK = 576;             // latent + rotary dimensions of a key row
constexpr int kDV = 512;             // latent dimensions (the value row)
constexpr int kM = 128;              // query heads per CTA (the MMA's M rows)
constexpr int kQuarters = 4;         // value-dimension quarters (one per CTA)
constexpr int kDQ = kDV / kQuarters; // 128 value dimensions per CTA
constexpr int kThreads = 256;        // thread t <-> head t % 128 (tensor-memory lane), half t / 128
constexpr int kTT = 64;              // tokens per tile
constexpr int kStages = 3;
constexpr int kBlocks = kDK / 64;                // 9 column blocks of 64 dimensions
constexpr int kBlockBytes = kTT * 128;           // 8 KB
constexpr int kTileBytes = kBlocks * kBlockBytes;  // 72 KB
constexpr int kSmem = 1024 + kStages * kTileBytes;  // (+ the 1024-byte alignment of the ring)
constexpr int kMaxChunk = 1024;                  // positions per CTA
constexpr uint32_t kCols = 512;
constexpr uint32_t kQCol = 0, kSCol = 288, kOCol = 384;
constexpr int kMaxMergeSplits = kStages * kTileBytes / (kM * 4);  // 432 (merge weights)
constexpr float kRescaleSlack = 8.f;             // log2 units
constexpr int kPRow = kDQ + 4;                   // partial row: m, l, 2 pad, o[128] (16-byte aligned)

static_assert(kQCol + kDK / 2 <= kSCol && kSCol + kTT <= kOCol && kOCol + kDQ <= kCols, "tmem");
static_assert(kTT == 64 && kThreads == 2 * kM, "two threads per head, 32 tokens each");

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
  long long wait_limit;  // clock cycles a wait in the tile loop may take (the drain waits longer)
  // the queries are complete before the preceding kernel starts (the decode step's own score
  // kernels precede this one): they are loaded while that kernel still runs
  int q_early;
};

__global__ void __launch_bounds__(kThreads, 1) mla_kernel(Args a, int chunk, int splits) {
  extern __shared__ __align__(1024) uint8_t mla_smem[];
  __shared__ int64_t s_off[kMaxChunk];
  __shared__ uint32_t s_valid[kMaxChunk / 32];  // bit j: position j of the slice is usable
  __shared__ __align__(8) uint64_t s_bar[3];     // S ready, P V done, drain
  __shared__ float s_half[2][kM];  // per-row exchange between the two halves (max, then l)
  __shared__ uint32_t s_tmem;
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // warps w and w + 4 share tensor-memory lanes 32 (w % 4) .. +31 (heads); half 0 takes tokens
  // 0-31 of a tile, the low half of the value dimensions and columns 0-159 of Q, half 1 the rest
  const int row = tid & (kM - 1), half = tid >> 7;
  const int hb = blockIdx.x / kQuarters, dq = blockIdx.x % kQuarters;
  const int split = blockIdx.y, b = blockIdx.z;
  const int n_hb = gridDim.x / kQuarters;
  const int max_len = a.max_pages * a.page_size;
  const uint32_t ring = (smem_u32(mla_smem) + 1023u) & ~1023u;
  const uint32_t bar_s = smem_u32(&s_bar[0]), bar_o = smem_u32(&s_bar[1]);
  const uint32_t bar_d = smem_u32(&s_bar[2]);

  if (tid == 0) {
    tc::mbar_init(bar_s, 1);
    tc::mbar_init(bar_o, 1);
    tc::mbar_init(bar_d, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(smem_u32(&s_tmem), kCols);
    tc::tmem_relinquish();
  }
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  // the query row of head `row` -> its tensor-memory lane, columns [0, 288): half 0 writes the
  // column groups 0-4, half 1 the groups 5-8 (24 independent 16-byte loads per round)
  auto load_q = [&](uint32_t tm) {
    const int head = hb * kM + row;
    const bool hv = head < a.h_q;
    const uint4* qrow = reinterpret_cast<const uint4*>(a.q + ((int64_t)b * a.h_q + (hv ? head : 0)) * kDK);
    const int g_begin = half ? 5 : 0, g_end = half ? kDK / 64 : 5;
#pragma unroll 1
    for (int g0 = g_begin; g0 < g_end; g0 += 3) {
      const int n = min(3, g_end - g0);  // (uniform over a warp)
      uint4 x[24];
#pragma unroll
      for (int u = 0; u < 24; ++u)
        x[u] = (hv && u < 8 * n) ? __ldg(qrow + g0 * 8 + u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int g3 = 0; g3 < 3; ++g3) {
        if (g3 >= n) break;
        uint32_t v[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          v[4 * u] = x[8 * g3 + u].x;
          v[4 * u + 1] = x[8 * g3 + u].y;
          v[4 * u + 2] = x[8 * g3 + u].z;
          v[4 * u + 3] = x[8 * g3 + u].w;
        }
        tc::tmem_st32(tm + lane_base + kQCol + 32 * (g0 + g3), v);
      }
    }
    tc::tmem_wait_st();
  };
  if (a.q_early) {
    tc::fence_before_sync();
    __syncthreads();  // the tensor-memory base address
    tc::fence_after_sync();
    load_q(s_tmem);
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
      int64_t off = -1;
      if (j < n_mine) {
        if (pos[u] < 0 || pos[u] >= max_len) raise_flag(2u);
        else if (pg[u] < 0 || (int64_t)pg[u] >= a.num_pages) raise_flag(1u);
        else off = (int64_t)pg[u] * a.page_stride + (int64_t)(pos[u] % a.page_size) * a.slot_stride;
      }
      s_off[j] = off;
      const unsigned m = __ballot_sync(0xffffffffu, off >= 0);
      if (lane == 0) s_valid[j >> 5] = m;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = s_tmem;

  // copies of a tile: 8 threads per row, thread q of a row takes the q-th 16-byte chunk of each
  // 128-byte column block (a warp instruction covers 128 contiguous bytes of each of its 4 rows)
  const int n_tiles = (n_mine + kTT - 1) / kTT;
  static_assert(kThreads / 8 == 32 && kTT % 32 == 0, "32 rows per copy pass");
  const int cp_row = tid >> 3, cp_q = tid & 7;
  auto issue = [&](int tl, int st) {
    const uint32_t stage = ring + st * kTileBytes;
#pragma unroll
    for (int p = 0; p < kTT / 32; ++p) {
      const int row = p * 32 + cp_row;
      const int j = tl * kTT + row;
      const int64_t off = j < n_mine ? s_off[j] : -1;
      const uint16_t* src = a.kv + (off >= 0 ? off : 0) + cp_q * 8;
      const uint32_t dst = stage + row * 128 + ((cp_q ^ (row & 7)) << 4);
#pragma unroll
      for (int blk = 0; blk < kBlocks; ++blk)
        cp_async16(dst + blk * kBlockBytes, src + blk * 64, off >= 0 ? 16 : 0);
    }
  };
  if (n_tiles > 0) issue(0, 0);
  cp_async_commit();

  if (!a.q_early) load_q(tmem);
  pdl_trigger();
  tc::fence_before_sync();
  __syncthreads();  // Q in tensor memory before the first MMA
  tc::fence_after_sync();

  const float scale_log2 = a.scale * 1.4426950408889634f;
  constexpr uint32_t kIdescS = tc::idesc_bf16(kM, kTT, false);
  constexpr uint32_t kIdescO = tc::idesc_bf16(kM, kDQ, true);
  float m_ref = -INFINITY, l_run = 0.f;
  bool ok = true;
  for (int i = 0; i < n_tiles; ++i) {
    // tile i + 1 goes to the stage of tile i - 2, whose P V completed before the previous
    // iteration's S: the copies are issued while P V of tile i - 1 still runs
    if (i + 1 < n_tiles) issue(i + 1, (i + 1) % kStages);
    cp_async_commit();
    cp_async_wait<1>();  // tile i (all but the newest group)
    tc::fence_proxy_async_smem();
    // P V of the previous tile done: S / P and O are free (and every thread's copies of tile i
    // are in once the barrier below passes)
    const bool w = i == 0 || tc::mbar_wait(bar_o, (i - 1) & 1, a.wait_limit);
    if (__syncthreads_or(!w)) {
      ok = false;
      break;
    }
    const uint32_t stage = ring + (i % kStages) * kTileBytes;
    if (tid == 0) {
      tc::fence_after_sync();
      // S = Q K^T: 36 steps of 16 dimensions; step kk reads 32 bytes at (kk % 4) * 32 of the
      // 128-byte rows of column block kk / 4. Fully unrolled, each descriptor the stage's plus a
      // constant (the address field holds the shared-memory address / 16 and cannot carry): the
      // issuing thread keeps up with the tensor cores
      const uint64_t b0 = tc::sw128_desc(stage, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < kDK / 16; ++kk)
        tc::mma_ts(tmem + kSCol, tmem + kQCol + kk * 8,
                   b0 + (uint64_t)(((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4), kIdescS,
                   kk > 0);
      tc::mma_commit(bar_s);
    }
    {
      const bool w = tc::mbar_wait(bar_s, i & 1, a.wait_limit);
      if (__syncthreads_or(!w)) {
        ok = false;
        break;
      }
    }
    tc::fence_after_sync();
    uint32_t sr[32];
    tc::tmem_ld32(tmem + lane_base + kSCol + 32 * half, sr);
    tc::tmem_wait_ld();
    const uint32_t vm = s_valid[2 * i + half];
    float x[32];
    float mt = -INFINITY;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      x[c] = ((vm >> c) & 1u) ? __uint_as_float(sr[c]) * scale_log2 : -INFINITY;
      mt = fmaxf(mt, x[c]);
    }
    // the row maximum over both halves; every S read is complete before P overwrites it
    s_half[half][row] = mt;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    mt = fmaxf(s_half[0][row], s_half[1][row]);
    // lazy rescale: the weights are taken relative to m_ref, which moves only when a row's
    // maximum exceeds it by more than the slack (weights stay <= 2^8)
    const bool first = m_ref == -INFINITY;
    const bool grow = mt > m_ref + kRescaleSlack;
    const bool resc = grow && !first;  // O holds earlier weights relative to the old m_ref
    const float m_new = grow ? mt : m_ref;
    const float corr = resc ? fast_exp2(m_ref - m_new) : 1.f;
    if (__any_sync(0xffffffffu, resc)) {  // this half's 64 columns of O
#pragma unroll 1
      for (int c = 0; c < kDQ / 64; ++c) {
        uint32_t o[32];
        const uint32_t col = kOCol + 64 * half + 32 * c;
        tc::tmem_ld32(tmem + lane_base + col, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
        tc::tmem_st32(tmem + lane_base + col, o);
      }
    }
    l_run *= corr;  // (this half's share of the row sum)
    m_ref = m_new;
    uint32_t ph[16], pl[16];
    float lsum = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float p0 = x[2 * e] == -INFINITY ? 0.f : fast_exp2(x[2 * e] - m_ref);
      const float p1 = x[2 * e + 1] == -INFINITY ? 0.f : fast_exp2(x[2 * e + 1] - m_ref);
      lsum += p0 + p1;
      const uint32_t h = pack_bf16x2(p0, p1);
      ph[e] = h;
      pl[e] = pack_bf16x2(p0 - bf16_lo(h), p1 - bf16_hi(h));
    }
    l_run += lsum;
    tc::tmem_st16(tmem + lane_base + kSCol + 16 * half, ph);
    tc::tmem_st16(tmem + lane_base + kSCol + 32 + 16 * half, pl);
    tc::tmem_wait_st();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      tc::fence_after_sync();
      // O += P V: K = 16 tokens per step; B = rows 16 kk.. of the quarter's two column blocks
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < kTT / 16; ++kk) {
          const uint64_t bd = tc::sw128_desc(stage + 2 * dq * kBlockBytes + kk * 16 * 128,
                                             kBlockBytes, 1024);
          tc::mma_ts(tmem + kOCol, tmem + kSCol + 32 * part + kk * 8, bd, kIdescO,
                     i > 0 || part > 0 || kk > 0);
        }
      tc::mma_commit(bar_o);
    }
  }
  if (ok && n_tiles > 0) {
    const bool w = tc::mbar_wait(bar_o, (n_tiles - 1) & 1, a.wait_limit);
    if (__syncthreads_or(!w)) ok = false;
    tc::fence_after_sync();
  }
  cp_async_wait<0>();
  // every MMA issued has completed before the tensor memory is read for the last time and freed
  if (tid == 0) tc::mma_commit(bar_d);
  if (__syncthreads_or(!tc::mbar_wait(bar_d, 0))) ok = false;
  tc::fence_after_sync();
  if (!ok && tid == 0) raise_flag(JSSA_DEVERR_TIMEOUT);

  // row sum over both halves
  s_half[half][row] = l_run;
  __syncthreads();
  const float l_tot = s_half[0][row] + s_half[1][row];
  const int head = hb * kM + row;
  const bool hv = head < a.h_q && ok;
  const bool have_o = n_tiles > 0 && ok;
  uint16_t* orow = a.out + ((int64_t)b * a.h_q + head) * kDV + dq * kDQ;
  const int64_t blk = ((int64_t)b * n_hb + hb) * kQuarters + dq;
  const int64_t n_blocks = (int64_t)a.batch * n_hb * kQuarters;
  int* tickets = reinterpret_cast<int*>(a.ws);
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.ws) +
                                         ((n_blocks * 4 + 255) / 256) * 256);
  float* prow = part + ((blk * splits + split) * kM + row) * kPRow;
  if (splits == 1) {
    const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
#pragma unroll 1
    for (int c = 2 * half; c < 2 * half + 2; ++c) {  // this half's 64 value dimensions
      uint32_t o[32];
      if (have_o) {
        tc::tmem_ld32(tmem + lane_base + kOCol + 32 * c, o);
        tc::tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
      if (hv)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          reinterpret_cast<uint4*>(orow + 32 * c)[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
    }
  } else {
    // partial [m (log2 units), l, -, -, o[128]] of this split (16-byte stores), then a ticket
    float4* p4 = reinterpret_cast<float4*>(prow);
    if (half == 0) __stcg(p4, make_float4(m_ref, l_tot, 0.f, 0.f));
#pragma unroll 1
    for (int c = 2 * half; c < 2 * half + 2; ++c) {
      uint32_t o[32];
      if (have_o) {
        tc::tmem_ld32(tmem + lane_base + kOCol + 32 * c, o);
        tc::tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0u;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e)
        __stcg(p4 + 1 + 8 * c + e, make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                               __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3])));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kCols);
  }
  if (splits == 1) return;

  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&tickets[blk], 1) == splits - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge: weights w = 2^(m - M) / L per (split, head) in shared memory (the ring is free), then
  // one weighted sum of independent loads per output element
  const float* p0 = part + blk * splits * kM * kPRow;
  const int64_t step = (int64_t)kM * kPRow;
  float* s_w = reinterpret_cast<float*>(mla_smem + (ring - smem_u32(mla_smem)));
  if (tid < kM) {  // row tid: the splits' (m, l) in batches of 8 independent loads, twice
    const float2* ml = reinterpret_cast<const float2*>(p0 + (int64_t)tid * kPRow);
    const int64_t st2 = step / 2;
    float mm = -INFINITY, l = 0.f;  // running maximum and the sum relative to it
    for (int sp0 = 0; sp0 < splits; sp0 += 8) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = sp0 + u < splits ? __ldcg(ml + (sp0 + u) * st2) : make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (v[u].x == -INFINITY) continue;
        if (v[u].x > mm) {
          l = l * fast_exp2(mm - v[u].x) + v[u].y;
          mm = v[u].x;
        } else {
          l += fast_exp2(v[u].x - mm) * v[u].y;
        }
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int sp0 = 0; sp0 < splits; sp0 += 8) {
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) m8[u] = sp0 + u < splits ? __ldcg(ml + (sp0 + u) * st2).x : -INFINITY;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (sp0 + u < splits)
          s_w[(sp0 + u) * kM + tid] = m8[u] != -INFINITY ? fast_exp2(m8[u] - mm) * inv : 0.f;
    }
  }
  __syncthreads();
  // 4 consecutive dimensions per task, consecutive threads on consecutive 16-byte pieces of a
  // row; 8 tasks unrolled so that their loads are in flight together
  constexpr int kTasks = kM * kDQ / 4;
#pragma unroll 1
  for (int e0 = 0; e0 < kTasks; e0 += 8 * kThreads) {
    float4 acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int sp = 0; sp < splits; ++sp) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = e0 + u * kThreads + tid, row = e / (kDQ / 4), d4 = e % (kDQ / 4);
        v[u] = __ldcg(reinterpret_cast<const float4*>(p0 + sp * step + (int64_t)row * kPRow + 4) + d4);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = e0 + u * kThreads + tid, row = e / (kDQ / 4);
        const float w = s_w[sp * kM + row];
        acc[u].x += w * v[u].x;
        acc[u].y += w * v[u].y;
        acc[u].z += w * v[u].z;
        acc[u].w += w * v[u].w;
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * kThreads + tid, row = e / (kDQ / 4), d4 = e % (kDQ / 4);
      const int h = hb * kM + row;
      if (h < a.h_q)
        *reinterpret_cast<uint2*>(a.out + ((int64_t)b * a.h_q + h) * kDV + dq * kDQ + 4 * d4) =
            make_uint2(pack_bf16x2(acc[u].x, acc[u].y), pack_bf16x2(acc[u].z, acc[u].w));
    }
  }
  if (tid == 0) tickets[blk] = 0;
}

}  // namespace mla_detail

int mla_tickets_per_sequence(int h_q) {
  using namespace mla_detail;
  return ((h_q + kM - 1) / kM) * kQuarters;
}

MlaPlan plan_mla(int batch, int h_q, int budget) {
  using namespace mla_detail;
  MlaPlan p;
  const int blocks = batch * ((h_q + kM - 1) / kM) * kQuarters;
  int splits = num_sms() / (blocks > 0 ? blocks : 1);  // one CTA per SM
  const int max_splits = (budget + kTT - 1) / kTT;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int chunk = (budget + splits - 1) / splits;
  chunk = (chunk + kTT - 1) / kTT * kTT;
  const int min_chunk = (budget + kMaxMergeSplits - 1) / kMaxMergeSplits;  // the merge buffer
  if (chunk < min_chunk) chunk = (min_chunk + kTT - 1) / kTT * kTT;
  if (chunk > kMaxChunk) chunk = kMaxChunk;
  splits = (budget + chunk - 1) / chunk;
  if (splits > kMaxMergeSplits) splits = 0;  // budget above kMaxMergeSplits * kMaxChunk
  p.splits = splits;
  p.chunk = chunk;
  p.ws_bytes = splits > 1 ? (((size_t)blocks * 4 + 255) / 256) * 256 +
                                (size_t)blocks * splits * kM * kPRow * sizeof(float)
                          : 0;
  return p;
}

cudaError_t launch_mla(const uint16_t* q, const uint16_t* kv, int64_t page_stride,
                       int64_t slot_stride, const int32_t* block_table, int max_pages,
                       const int32_t* idx, const int32_t* count, int batch, int h_q, int budget,
                       int64_t num_pages, int page_size, float scale, uint16_t* out, void* ws,
                       const MlaPlan& plan, bool pdl, cudaStream_t s, bool q_early) {
  using namespace mla_detail;
  if (batch == 0) return cudaSuccess;
  static_assert(kSmem - 1024 >= kMaxMergeSplits * kM * 4, "merge buffer");
  cudaError_t e = configure_kernel((const void*)mla_kernel, kSmem, false);
  if (e != cudaSuccess) return e;
  Args a = {q, kv, page_stride, slot_stride, block_table, max_pages, idx, count, batch, h_q,
            budget, num_pages, page_size, scale, out, ws, tc_wait_limit(), q_early ? 1 : 0};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(((h_q + kM - 1) / kM) * kQuarters, plan.splits, batch);
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
