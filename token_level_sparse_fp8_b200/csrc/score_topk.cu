// Score + top-B (JSSA summary, eq. (1) and section 3.1 steps 1-2; JSSA README, section 4:
// jssa_budget tokens per decode step and KV head).
//
// One thread-block cluster per (sequence, KV head). CTA c of the cluster owns tokens
// [c*chunk, (c+1)*chunk) of the sequence:
//   1. p = M_h qbar (qbar = mean of the G query heads of KV head h), fp32, in shared memory;
//   2. stream the chunk's FP8 scoring rows (page-table indexed, 16-byte non-allocating loads,
//      8 independent loads per thread in flight) and keep every score as an order-preserving
//      32-bit key in shared memory -- scores never go to HBM;
//   3. exact radix select of the budget-th largest key over the whole cluster: three digit
//      passes (11, 11, 10 bits); each CTA histograms its own keys, the histograms are summed
//      through distributed shared memory (each CTA reduces one slice of the bins), and every CTA
//      finds the threshold digit from the slice totals;
//   4. keys above the threshold are selected, keys equal to it are taken in position order up to
//      the remaining quota (ties go to the lower position); a cluster-wide prefix of the per-CTA
//      counts gives each CTA its output offset, so the index set comes out in ascending order.
// When seq_len <= budget every position is selected without scoring.
#include "common.cuh"

namespace jssa {

namespace score_detail {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 8;  // 16-byte loads in flight per thread
constexpr int kBins = 2048;

__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive prefix sum over the block (in thread order); also returns the block total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* s_warp,
                                                         uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  uint32_t base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t t = s_warp[w];
    base += (w < warp) ? t : 0u;
    tot += t;
  }
  __syncthreads();
  total = tot;
  return base + x - v;
}

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* s_warp) {
  uint32_t tot;
  block_exclusive_scan(v, s_warp, tot);
  return tot;
}

template <int R>
__device__ __forceinline__ float dot16(const uint4& v, const float* p) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 a = e4m3x2_to_f2((uint16_t)(w[i] & 0xFFFFu));
    const float2 b = e4m3x2_to_f2((uint16_t)(w[i] >> 16));
    acc = fmaf(a.x, p[4 * i + 0], acc);
    acc = fmaf(a.y, p[4 * i + 1], acc);
    acc = fmaf(b.x, p[4 * i + 2], acc);
    acc = fmaf(b.y, p[4 * i + 3], acc);
  }
  return acc;
}

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 3)
    score_topk_kernel(const uint16_t* __restrict__ q, const float* __restrict__ basis,
                      const uint8_t* __restrict__ score_cache,
                      const int32_t* __restrict__ block_table, int max_pages,
                      const int32_t* __restrict__ seq_lens, int h_q, int h_kv, int64_t num_pages,
                      int page_size, int budget, int chunk, int32_t* __restrict__ idx,
                      int32_t* __restrict__ count) {
  constexpr int PPT = R / 16;     // 16-byte pieces per token row
  constexpr int TPG = 32 / PPT;   // tokens covered by one warp-wide load
  static_assert(PPT >= 1 && PPT <= 8, "rank");

  extern __shared__ uint32_t dyn[];
  uint32_t* s_key = dyn;                                      // [chunk]
  int32_t* s_page = reinterpret_cast<int32_t*>(dyn + chunk);  // [chunk / page_size + 1]
  __shared__ float s_qbar[D];
  __shared__ float s_p[R];
  __shared__ uint32_t s_hist[kBins];
  __shared__ uint32_t s_red[kBins];
  __shared__ uint32_t s_tot;
  __shared__ uint32_t s_cnt[2];
  __shared__ uint32_t s_warp[kWarps];
  __shared__ int32_t s_info[4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = blockIdx.y;
  const int b = pair / h_kv, h = pair % h_kv;
  const int G = h_q / h_kv;
  const uint32_t crank = cluster_rank();
  const uint32_t C = cluster_size();
  const int max_len = max_pages * page_size;

  int L = seq_lens[b];
  if (L < 0 || L > max_len) {
    if (tid == 0 && crank == 0) raise_flag(4u);
    L = L < 0 ? 0 : max_len;
  }
  int32_t* out_idx = idx + (int64_t)pair * budget;
  const int start = (int)crank * chunk;

  if (L <= budget) {
    // Every position is selected: no scores are needed.
    const int per = (budget + (int)C - 1) / (int)C;
    const int j0 = (int)crank * per, j1 = min(budget, j0 + per);
    for (int j = j0 + tid; j < j1; j += kThreads) out_idx[j] = j < L ? j : -1;
    if (crank == 0 && tid == 0) count[pair] = L;
    return;
  }

  // ---- 1. projected group-mean query --------------------------------------------------------
  const uint16_t* qh = q + ((int64_t)b * h_q + (int64_t)h * G) * D;
  for (int i = tid; i < D; i += kThreads) {
    float acc = 0.f;
    for (int g = 0; g < G; ++g) acc += bf16_to_f(qh[(int64_t)g * D + i]);
    s_qbar[i] = acc / (float)G;
  }
  __syncthreads();
  {
    constexpr int TPJ = kThreads / R;  // threads per output
    constexpr int DPT = D / TPJ;
    static_assert(TPJ >= 1 && TPJ <= 32 && D % TPJ == 0, "projection split");
    const int j = tid / TPJ, sub = tid % TPJ;
    const float* mrow = basis + ((int64_t)h * R + j) * D + sub * DPT;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < DPT; ++i) acc = fmaf(mrow[i], s_qbar[sub * DPT + i], acc);
#pragma unroll
    for (int o = TPJ / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (sub == 0) s_p[j] = acc;
  }

  // ---- 2. page list of this chunk ------------------------------------------------------------
  const int n_local = max(0, min(chunk, L - start));
  const int n_pages_local = (n_local + page_size - 1) / page_size;
  const int32_t* bt = block_table + (int64_t)b * max_pages + start / page_size;
  for (int i = tid; i < n_pages_local; i += kThreads) {
    int32_t pg = bt[i];
    if (pg < 0 || (int64_t)pg >= num_pages) {
      raise_flag(1u);
      pg = -1;
    }
    s_page[i] = pg;
  }
  __syncthreads();

  float p_reg[16];
  {
    const int piece = lane % PPT;
#pragma unroll
    for (int e = 0; e < 16; ++e) p_reg[e] = s_p[piece * 16 + e];
  }

  // The scoring rows of the new token are written by the preceding store kernel.
  pdl_wait();

  // ---- 3. scores -> keys in shared memory ----------------------------------------------------
  const int n_groups = (n_local + TPG - 1) / TPG;
  const int64_t head_off = (int64_t)h * page_size * R;
  const int64_t page_bytes = (int64_t)h_kv * page_size * R;
  const int tok_in_group = lane / PPT;
  const int piece = lane % PPT;
  for (int g0 = warp * kUnroll; g0 < n_groups; g0 += kWarps * kUnroll) {
    uint4 v[kUnroll];
    int tok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      tok[u] = (g0 + u) * TPG + tok_in_group;
      int pg = -1;
      if (tok[u] < n_local) pg = s_page[tok[u] / page_size];
      if (pg >= 0) {
        const uint8_t* src = score_cache + (int64_t)pg * page_bytes + head_off +
                             (int64_t)(tok[u] % page_size) * R + piece * 16;
        v[u] = ld_stream_v4(src);
      } else {
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (tok[u] >= n_local) tok[u] = -1;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float s = dot16<R>(v[u], p_reg);
#pragma unroll
      for (int o = 1; o < PPT; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (piece == 0 && tok[u] >= 0) s_key[tok[u]] = score_key(s);
    }
  }
  __syncthreads();

  // ---- 4. cluster-wide radix select of the budget-th largest key -----------------------------
  uint32_t prefix = 0, pmask = 0;
  int want = budget;  // rank (1-based, from the top) of the threshold among keys matching prefix
  const uint32_t hist_addr = smem_u32(s_hist);
  const uint32_t red_addr = smem_u32(s_red);
  const uint32_t tot_addr = smem_u32(&s_tot);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    for (int i = tid; i < nb; i += kThreads) s_hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n_local; i += kThreads) {
      const uint32_t key = s_key[i];
      if ((key & pmask) == prefix) atomicAdd(&s_hist[(key >> shift) & (nb - 1)], 1u);
    }
    cluster_sync();  // every histogram of the cluster is complete
    const int per = nb / (int)C;
    uint32_t part = 0;
    for (int j = tid; j < per; j += kThreads) {
      uint32_t sum = 0;
      const uint32_t off = (uint32_t)((int)crank * per + j) * 4u;
      for (uint32_t r = 0; r < C; ++r) sum += ld_cluster_u32(map_rank(hist_addr + off, r));
      s_red[j] = sum;
      part += sum;
    }
    part = block_sum(part, s_warp);
    if (tid == 0) s_tot = part;
    cluster_sync();  // every slice sum and slice total is published
    if (warp == 0) {
      // slice totals, top slice first
      const uint32_t r_lane = C - 1 - (uint32_t)lane;
      uint32_t t = (lane < (int)C) ? ld_cluster_u32(map_rank(tot_addr, r_lane)) : 0u;
      uint32_t incl = t;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - t;
      const unsigned hit = __ballot_sync(0xffffffffu, lane < (int)C && excl < (uint32_t)want &&
                                                          incl >= (uint32_t)want);
      // lane index of the slice holding the threshold (always found for consistent counts; the
      // fallback keeps every cluster address valid if the counts were ever inconsistent)
      const int sl = hit ? __ffs(hit) - 1 : 0;
      const uint32_t above_slice = __shfl_sync(0xffffffffu, excl, sl);
      const uint32_t rank_sl = C - 1 - (uint32_t)sl;
      // bins of that slice, highest first: lane i takes bins [per - (i+1)*bpl, per - i*bpl)
      const int bpl = (per + 31) / 32;
      const int hi = per - lane * bpl;
      const int lo = max(0, hi - bpl);
      uint32_t c = 0;
      for (int j = lo; j < hi; ++j) c += ld_cluster_u32(map_rank(red_addr + (uint32_t)j * 4u, rank_sl));
      uint32_t incl2 = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl2, o);
        if (lane >= o) incl2 += y;
      }
      const uint32_t excl2 = above_slice + incl2 - c;
      const unsigned hit2 = __ballot_sync(0xffffffffu, hi > lo && excl2 < (uint32_t)want &&
                                                           excl2 + c >= (uint32_t)want);
      const int ln = hit2 ? __ffs(hit2) - 1 : 0;
      if (lane == 0 && (!hit || !hit2)) raise_flag(8u);
      if (lane == ln) {
        uint32_t run = excl2;
        int bin = lo;
        for (int j = hi - 1; j >= lo; --j) {
          const uint32_t cj = ld_cluster_u32(map_rank(red_addr + (uint32_t)j * 4u, rank_sl));
          if (run + cj >= (uint32_t)want) { bin = j; break; }
          run += cj;
        }
        s_info[0] = (int)rank_sl * per + bin;
        s_info[1] = (int)run;  // keys (matching the prefix) in strictly higher bins
      }
    }
    __syncthreads();
    const uint32_t digit = (uint32_t)s_info[0];
    want -= s_info[1];
    prefix |= digit << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    __syncthreads();
  }
  const uint32_t thr = prefix;  // the budget-th largest key; `want` keys equal to it are taken

  // ---- 5. emit the index set in ascending position order -------------------------------------
  const int kpt = (n_local + kThreads - 1) / kThreads;
  const int r0 = min(n_local, tid * kpt), r1 = min(n_local, r0 + kpt);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = r0; i < r1; ++i) {
    const uint32_t key = s_key[i];
    n_gt += key > thr;
    n_eq += key == thr;
  }
  uint32_t tot_gt, tot_eq;
  block_exclusive_scan(n_gt, s_warp, tot_gt);
  const uint32_t eq_base = block_exclusive_scan(n_eq, s_warp, tot_eq);
  if (tid == 0) {
    s_cnt[0] = tot_gt;
    s_cnt[1] = tot_eq;
  }
  cluster_sync();  // per-CTA counts are published
  if (tid == 0) {
    const uint32_t cnt_addr = smem_u32(s_cnt);
    uint32_t rem = (uint32_t)want, offset = 0, my_take = 0;
    for (uint32_t r = 0; r < C; ++r) {
      const uint32_t gt = ld_cluster_u32(map_rank(cnt_addr, r));
      const uint32_t eq = ld_cluster_u32(map_rank(cnt_addr + 4u, r));
      const uint32_t take = eq < rem ? eq : rem;
      rem -= take;
      if (r < crank) offset += gt + take;
      if (r == crank) my_take = take;
    }
    s_info[2] = (int)offset;
    s_info[3] = (int)my_take;
  }
  __syncthreads();
  const uint32_t offset = (uint32_t)s_info[2], my_take = (uint32_t)s_info[3];
  uint32_t n_sel = 0;
  {
    uint32_t seen = eq_base;
    for (int i = r0; i < r1; ++i) {
      const uint32_t key = s_key[i];
      if (key > thr) ++n_sel;
      else if (key == thr) { n_sel += seen < my_take; ++seen; }
    }
  }
  uint32_t tot_sel;
  uint32_t pos = offset + block_exclusive_scan(n_sel, s_warp, tot_sel);
  {
    uint32_t seen = eq_base;
    for (int i = r0; i < r1; ++i) {
      const uint32_t key = s_key[i];
      bool take = key > thr;
      if (key == thr) { take = seen < my_take; ++seen; }
      if (take && pos < (uint32_t)budget) out_idx[pos++] = start + i;
    }
  }
  if (crank == 0 && tid == 0) count[pair] = budget;
  pdl_trigger();
  cluster_sync();  // no CTA leaves while another may still read its shared memory
}

template <int D, int R>
cudaError_t launch_t(const ScorePlan& plan, int pairs, bool pdl, cudaStream_t s, const uint16_t* q,
                     const float* basis, const uint8_t* score_cache, const int32_t* block_table,
                     int max_pages, const int32_t* seq_lens, int h_q, int h_kv, int64_t num_pages,
                     int page_size, int budget, int32_t* idx, int32_t* count) {
  auto kern = score_topk_kernel<D, R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem);
  if (e != cudaSuccess) return e;
  if (plan.cluster > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.cluster, pairs, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = plan.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, kern, q, basis, score_cache, block_table, max_pages, seq_lens, h_q,
                         h_kv, num_pages, page_size, budget, plan.chunk, idx, count);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace score_detail

ScorePlan plan_score(int pairs, int max_seq_len, int page_size) {
  ScorePlan p;
  // tokens per CTA must be a multiple of the page size (so a CTA's pages start on a page) and of
  // 64 (whole warp-wide loads)
  int align = 64;
  while (align % page_size) align += 64;
  int c = 1;
  while (c < kMaxClusterCtas && (long long)c * kScoreChunkTarget < max_seq_len) c <<= 1;
  // more CTAs per (sequence, head) while the GPU would otherwise be under-filled
  const int want_ctas = 2 * num_sms();
  while (c < kMaxClusterCtas && (long long)pairs * c < want_ctas && max_seq_len / (2 * c) >= 1024)
    c <<= 1;
  int chunk = (max_seq_len + c - 1) / c;
  chunk = (chunk + align - 1) / align * align;
  p.cluster = c;
  p.chunk = chunk;
  p.smem = (size_t)chunk * 4 + (size_t)(chunk / page_size + 1) * 4;
  return p;
}

cudaError_t launch_score_topk(const uint16_t* q, const float* basis, const uint8_t* score_cache,
                              const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                              int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                              int page_size, int budget, int32_t* idx, int32_t* count, bool pdl,
                              cudaStream_t s) {
  const int pairs = batch * h_kv;
  if (pairs == 0) return cudaSuccess;
  const ScorePlan plan = plan_score(pairs, max_pages * page_size, page_size);
  if (d == 128 && r == 32)
    return score_detail::launch_t<128, 32>(plan, pairs, pdl, s, q, basis, score_cache, block_table, max_pages,
                             seq_lens, h_q, h_kv, num_pages, page_size, budget, idx, count);
  if (d == 128 && r == 64)
    return score_detail::launch_t<128, 64>(plan, pairs, pdl, s, q, basis, score_cache, block_table, max_pages,
                             seq_lens, h_q, h_kv, num_pages, page_size, budget, idx, count);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
