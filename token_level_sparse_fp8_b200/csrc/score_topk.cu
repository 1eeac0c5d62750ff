// Score + top-B (JSSA summary, eq. (1) and section 3.1 steps 1-2; JSSA README, section 4:
// jssa_budget tokens per decode step and KV head).
//
// One thread-block cluster per (sequence, KV head). CTA c of the cluster owns tokens
// [c*chunk, (c+1)*chunk) of the sequence:
//   1. p = M_h qbar (qbar = mean of the G query heads of KV head h), fp32, in shared memory;
//   2. stream the chunk's FP8 scoring rows (page-table indexed, 16-byte non-allocating loads,
//      8 independent loads per thread in flight) and keep every score as an order-preserving
//      32-bit key in shared memory -- scores never go to HBM. The E4M3 codes are widened with
//      integer operations (sign and the 7 exponent/mantissa bits are moved into an fp32 bit
//      pattern whose value is the code's value times 2^-120); the power of two is folded into p,
//      together with a per-head power-of-two scale that keeps every product finite, so each key
//      orders exactly as the score would. The histogram of the first radix digit is built in the
//      same loop;
//   3. exact radix select of the budget-th largest key over the whole cluster: up to three
//      digit passes (11, 11, 10 bits), stopping early once the threshold bin is taken whole.
//      Each CTA histograms its own keys, every CTA sums one slice of the bins across the cluster
//      through distributed shared memory, and every CTA locates the threshold digit from the
//      slice totals;
//   4. keys above the threshold are selected, keys equal to it are taken in position order up to
//      the remaining quota (ties go to the lower position); warp ballots give each key its rank
//      inside the CTA and a cluster-wide prefix of the per-CTA counts gives the CTA's offset, so
//      the index set comes out in ascending order.
// When seq_len <= budget every position is selected without scoring.
#include "common.cuh"

namespace jssa {

namespace score_detail {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 8;  // 16-byte loads in flight per thread
constexpr int kBins = 2048;

template <typename T>
__device__ __forceinline__ T* remote(T* p, uint32_t rank) {
  return static_cast<T*>(__cluster_map_shared_rank(p, rank));
}

// fp32 whose value is (E4M3 code in the top byte of x) * 2^-120: sign stays in bit 31, the
// exponent and mantissa bits move down by 4 into the low exponent / high mantissa positions.
__device__ __forceinline__ float e4m3_top_byte_scaled(uint32_t x) {
  return __uint_as_float((x & 0x80000000u) | ((x & 0x7F000000u) >> 4));
}

__device__ __forceinline__ float dot16(const uint4& v, const float* p) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc0 = fmaf(e4m3_top_byte_scaled(w[i] << 24), p[4 * i + 0], acc0);
    acc1 = fmaf(e4m3_top_byte_scaled(w[i] << 16), p[4 * i + 1], acc1);
    acc0 = fmaf(e4m3_top_byte_scaled(w[i] << 8), p[4 * i + 2], acc0);
    acc1 = fmaf(e4m3_top_byte_scaled(w[i]), p[4 * i + 3], acc1);
  }
  return acc0 + acc1;
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

__device__ __forceinline__ uint32_t block_sum(uint32_t v, uint32_t* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) s_warp[warp] = v;
  __syncthreads();
  uint32_t t = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += s_warp[w];
  __syncthreads();
  return t;
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

  extern __shared__ uint32_t score_dyn[];
  uint32_t* s_key = score_dyn;                                      // [chunk]
  int32_t* s_page = reinterpret_cast<int32_t*>(score_dyn + chunk);  // [chunk / page_size + 1]
  __shared__ float s_qbar[D];
  __shared__ float s_p[R];
  __shared__ uint32_t s_hist[kBins];
  __shared__ uint32_t s_red[kBins];
  __shared__ uint32_t s_tot;
  __shared__ uint32_t s_cnt[2];       // keys above / equal to the threshold in this CTA
  __shared__ uint32_t s_warp[kWarps];
  __shared__ uint32_t s_wgt[kWarps], s_weq[kWarps];
  __shared__ int32_t s_info[4];
  __shared__ float s_pmax;

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
  for (int i = tid; i < kBins; i += kThreads) s_hist[i] = 0u;
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
  if (warp == 0) {
    float m = 0.f;
    for (int j = lane; j < R; j += 32) m = fmaxf(m, fabsf(s_p[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_pmax = m;
  }
  __syncthreads();

  // p scaled by 2^(120 - E): the decoded codes carry a factor 2^-120, and E >= 0 keeps
  // |p'| * 448 * R far below the float range. A power-of-two scale is exact, so the keys order
  // exactly like the unscaled scores.
  float p_reg[16];
  {
    const int ex = (int)((__float_as_uint(s_pmax) >> 23) & 0xFF) - 127;  // floor(log2 max|p|)
    const int E = max(0, ex + 7);
    const float scale = __uint_as_float((uint32_t)(127 + 120 - E) << 23);
    const int piece = lane % PPT;
#pragma unroll
    for (int e = 0; e < 16; ++e) p_reg[e] = s_p[piece * 16 + e] * scale;
  }

  // The scoring rows of the new token are written by the preceding store kernel.
  pdl_wait();

  // ---- 3. scores -> keys in shared memory, first-digit histogram -----------------------------
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
      float s = dot16(v[u], p_reg);
#pragma unroll
      for (int o = 1; o < PPT; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (piece == 0 && tok[u] >= 0) {
        const uint32_t key = score_key(s);
        s_key[tok[u]] = key;
        atomicAdd(&s_hist[key >> 21], 1u);
      }
    }
  }
  __syncthreads();

  // ---- 4. cluster-wide radix select of the budget-th largest key -----------------------------
  uint32_t prefix = 0, pmask = 0;
  int want = budget;  // rank (1-based, from the top) of the threshold among keys matching prefix
  uint32_t thr = 0;
  bool resolved = false;
#pragma unroll 1
  for (int pass = 0; pass < 3 && !resolved; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    if (pass > 0) {
      for (int i = tid; i < nb; i += kThreads) s_hist[i] = 0u;
      __syncthreads();
      for (int i = tid; i < n_local; i += kThreads) {
        const uint32_t key = s_key[i];
        if ((key & pmask) == prefix) atomicAdd(&s_hist[(key >> shift) & (nb - 1)], 1u);
      }
    }
    cluster_sync();  // every histogram of the cluster is complete
    const int per = nb / (int)C;
    uint32_t part = 0;
    for (int j = tid; j < per; j += kThreads) {
      const int bin = (int)crank * per + j;
      uint32_t sum = 0;
      for (uint32_t r = 0; r < C; ++r) sum += *remote(&s_hist[bin], r);
      s_red[j] = sum;
      part += sum;
    }
    part = block_sum(part, s_warp);
    if (tid == 0) s_tot = part;
    cluster_sync();  // every slice sum and slice total is published
    if (warp == 0) {
      // slice totals, top slice first; lane i holds slice C-1-i
      const uint32_t r_lane = C - 1 - (uint32_t)lane;
      const uint32_t t = (lane < (int)C) ? *remote(&s_tot, r_lane) : 0u;
      const uint32_t incl = warp_incl_scan(t, lane);
      const uint32_t excl = incl - t;
      const unsigned hit = __ballot_sync(0xffffffffu, lane < (int)C && excl < (uint32_t)want &&
                                                          incl >= (uint32_t)want);
      // (always found for consistent counts; the fallback keeps every address in the cluster)
      const int sl = hit ? __ffs(hit) - 1 : 0;
      const uint32_t above_slice = __shfl_sync(0xffffffffu, excl, sl);
      const uint32_t rank_sl = C - 1 - (uint32_t)sl;
      const uint32_t* red = remote(s_red, rank_sl);
      // bins of that slice, highest first: lane i takes bins [per - (i+1)*bpl, per - i*bpl)
      const int bpl = (per + 31) / 32;
      const int hi = per - lane * bpl;
      const int lo = max(0, hi - bpl);
      uint32_t c = 0;
      for (int j = lo; j < hi; ++j) c += red[j];
      const uint32_t incl2 = warp_incl_scan(c, lane);
      const uint32_t excl2 = above_slice + incl2 - c;
      const unsigned hit2 = __ballot_sync(0xffffffffu, hi > lo && excl2 < (uint32_t)want &&
                                                           excl2 + c >= (uint32_t)want);
      const int ln = hit2 ? __ffs(hit2) - 1 : 0;
      if (lane == 0 && (!hit || !hit2)) raise_flag(8u);
      if (lane == ln) {
        uint32_t run = excl2, cnt = 0;
        int bin = lo;
        for (int j = hi - 1; j >= lo; --j) {
          const uint32_t cj = red[j];
          if (run + cj >= (uint32_t)want) { bin = j; cnt = cj; break; }
          run += cj;
        }
        s_info[0] = (int)rank_sl * per + bin;
        s_info[1] = (int)run;  // keys (matching the prefix) in strictly higher bins
        s_info[2] = (int)cnt;  // keys in the threshold bin
      }
    }
    __syncthreads();
    const uint32_t digit = (uint32_t)s_info[0];
    const int above = s_info[1], in_bin = s_info[2];
    __syncthreads();
    want -= above;
    prefix |= digit << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    if (want == in_bin) {
      // the whole threshold bin is selected: select every key >= its lowest key, no quota
      thr = prefix - 1u;  // prefix > 0: keys of finite scores are >= 0x00800000
      want = 0;
      resolved = true;
    } else if (pass == 2) {
      thr = prefix;
      resolved = true;
    }
  }

  // ---- 5. emit the index set in ascending position order -------------------------------------
  // warp w owns positions [w*seg, (w+1)*seg) of the chunk, walked 32 at a time (lane = position)
  const int seg = ((n_local + kWarps - 1) / kWarps + 31) & ~31;
  const int w0 = min(n_local, warp * seg), w1 = min(n_local, w0 + seg);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < w1 ? s_key[i] : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, i < w1 && key > thr));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < w1 && key == thr));
  }
  if (lane == 0) {
    s_wgt[warp] = n_gt;
    s_weq[warp] = n_eq;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kWarps; ++w) {
      g += s_wgt[w];
      e += s_weq[w];
    }
    s_cnt[0] = g;
    s_cnt[1] = e;
  }
  cluster_sync();  // per-CTA counts are published
  if (warp == 0) {
    // lane r < C holds CTA r's counts; the tie quota is handed out in rank (= position) order
    const uint32_t gt = lane < (int)C ? *remote(&s_cnt[0], (uint32_t)lane) : 0u;
    const uint32_t eq = lane < (int)C ? *remote(&s_cnt[1], (uint32_t)lane) : 0u;
    const uint32_t eq_before = warp_incl_scan(eq, lane) - eq;
    const uint32_t rem = (uint32_t)want > eq_before ? (uint32_t)want - eq_before : 0u;
    const uint32_t take = eq < rem ? eq : rem;
    const uint32_t sel = gt + take;
    const uint32_t sel_before = warp_incl_scan(sel, lane) - sel;
    if (lane == (int)crank) {
      s_info[2] = (int)sel_before;
      s_info[3] = (int)take;
    }
  }
  __syncthreads();
  const uint32_t cta_offset = (uint32_t)s_info[2], cta_take = (uint32_t)s_info[3];
  // this warp's quota of equal keys and output offset within the CTA
  uint32_t eq_before = 0, sel_before = 0;
  for (int w = 0; w < warp; ++w) {
    const uint32_t rem = cta_take > eq_before ? cta_take - eq_before : 0u;
    const uint32_t tk = s_weq[w] < rem ? s_weq[w] : rem;
    sel_before += s_wgt[w] + tk;
    eq_before += s_weq[w];
  }
  uint32_t eq_seen = eq_before;
  uint32_t pos = cta_offset + sel_before;
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < w1 ? s_key[i] : 0u;
    const bool is_eq = i < w1 && key == thr;
    const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool take = (i < w1 && key > thr) || (is_eq && eq_seen + __popc(eqm & lt) < cta_take);
    const unsigned selm = __ballot_sync(0xffffffffu, take);
    const uint32_t at = pos + __popc(selm & lt);
    if (take && at < (uint32_t)budget) out_idx[at] = start + i;
    pos += __popc(selm);
    eq_seen += __popc(eqm);
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
  cudaError_t e = configure_kernel((const void*)kern, (int)plan.smem, plan.cluster > 8);
  if (e != cudaSuccess) return e;
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
    return score_detail::launch_t<128, 32>(plan, pairs, pdl, s, q, basis, score_cache, block_table,
                                           max_pages, seq_lens, h_q, h_kv, num_pages, page_size,
                                           budget, idx, count);
  if (d == 128 && r == 64)
    return score_detail::launch_t<128, 64>(plan, pairs, pdl, s, q, basis, score_cache, block_table,
                                           max_pages, seq_lens, h_q, h_kv, num_pages, page_size,
                                           budget, idx, count);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
