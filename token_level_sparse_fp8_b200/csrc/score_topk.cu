// Score + top-B (JSSA summary, eq. (1) and section 3.1 steps 1-2; JSSA README, section 4:
// jssa_budget tokens per decode step and KV head).
//
// One thread-block cluster per (sequence, KV head). CTA c of the cluster owns tokens
// [c*chunk, (c+1)*chunk) of the sequence:
//   1. p = M_h qbar (qbar = mean of the G query heads of KV head h), fp32. p is written as a sum
//      of 8 FP8 "digit" vectors with power-of-two column scales, p = sum_c 2^e_c D_c with each
//      D_c in E4M3 (digit c rounds what the earlier digits left over), which represents p to
//      ~2^-32 of its largest component;
//   2. stream the chunk's FP8 scoring rows (page-table indexed, 8-byte non-allocating loads,
//      16 independent loads per thread in flight). The codes are consumed as they are by the
//      tensor cores: one mma.sync m16n8k32 E4M3 x E4M3 -> fp32 per 16 tokens and 32 code bytes
//      multiplies the 16 rows by the 8 digit columns, and s = sum_c 2^e_c C[:, c]. (Widening the
//      codes on the CUDA cores costs ~3 instructions per byte and leaves this HBM-bound loop
//      issue-bound.) Every score is kept as an order-preserving 32-bit key in shared memory --
//      scores never go to HBM; the histogram of the key's top 11 bits is built in the same loop;
//   3. cluster round 1: every CTA sums one slice of the histogram bins across the cluster through
//      distributed shared memory; round 2: every CTA locates the bin that holds the budget-th
//      largest key (the threshold bin) from the slice totals;
//   4. every warp compacts its keys at or above the threshold bin -- the only keys that can be
//      selected -- into its own region of the workspace, in position order, with positions;
//   5. round 3, then all CTAs but rank 0 leave; rank 0 finds the exact budget-th largest key among
//      those candidates (two more radix digits of 11 and 10 bits, unless the threshold bin is
//      taken whole), takes every key above it and the equal keys in position order up to the
//      budget (ties go to the lower position), and writes the index set in ascending order.
// When seq_len <= budget every position is selected without scoring.
#include "common.cuh"

namespace jssa {

namespace score_detail {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnrollBytes = 64;  // bytes of scoring rows per lane in flight
constexpr int kBins = 2048;
constexpr int kDigits = 8;  // FP8 digit columns of p (the n = 8 of the mma)

template <typename T>
__device__ __forceinline__ T* remote(T* p, uint32_t rank) {
  return static_cast<T*>(__cluster_map_shared_rank(p, rank));
}

__device__ __forceinline__ void mma_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

// Bin of a histogram (`nb` bins, read through `at`) holding the want-th largest element counted
// from the top, given `above` elements in higher bins. Warp-wide; returns (bin, count of elements
// in strictly higher bins, count in the bin) on every lane.
template <typename At>
__device__ __forceinline__ void find_bin(At at, int nb, uint32_t above, uint32_t want, int lane,
                                         int& bin_out, uint32_t& above_out, uint32_t& cnt_out,
                                         bool& found) {
  const int bpl = (nb + 31) / 32;
  const int hi = nb - lane * bpl;
  const int lo = max(0, hi - bpl);
  uint32_t c = 0;
  for (int j = lo; j < hi; ++j) c += at(j);
  const uint32_t incl = warp_incl_scan(c, lane);
  const uint32_t excl = above + incl - c;
  const unsigned hit = __ballot_sync(0xffffffffu, hi > lo && excl < want && excl + c >= want);
  found = hit != 0;
  const int ln = hit ? __ffs(hit) - 1 : 0;
  int bin = 0;
  uint32_t run = 0, cnt = 0;
  if (lane == ln) {
    run = excl;
    bin = lo;
    for (int j = hi - 1; j >= lo; --j) {
      const uint32_t cj = at(j);
      if (run + cj >= want) { bin = j; cnt = cj; break; }
      run += cj;
    }
  }
  bin_out = __shfl_sync(0xffffffffu, bin, ln);
  above_out = __shfl_sync(0xffffffffu, run, ln);
  cnt_out = __shfl_sync(0xffffffffu, cnt, ln);
}

// Candidate regions: CTA c, warp w of a pair owns entries [(c*kWarps + w)*seg, +seg).
struct Cands {
  uint32_t* key;       // [pairs][C * kWarps * seg]
  int32_t* pos;        // [pairs][C * kWarps * seg]
  uint32_t* cnt;       // [pairs][kMaxClusterCtas * kWarps]
  int* attend_tickets; // [pairs] split-K tickets of the attention that follows, or null
};

__host__ __device__ inline int warp_seg(int chunk) { return ((chunk / kWarps) + 31) & ~31; }
__host__ __device__ inline size_t cand_bytes_counts(int pairs) {
  return ((size_t)pairs * kMaxClusterCtas * kWarps * 4 + 255) / 256 * 256;
}

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 3)
    score_topk_kernel(const uint16_t* __restrict__ q, const float* __restrict__ basis,
                      const uint8_t* __restrict__ score_cache,
                      const int32_t* __restrict__ block_table, int max_pages,
                      const int32_t* __restrict__ seq_lens, int h_q, int h_kv, int64_t num_pages,
                      int page_shift, int budget, int chunk, int32_t* __restrict__ idx,
                      int32_t* __restrict__ count, Cands cands) {
  constexpr int KB = R / 32;      // k-blocks of 32 codes
  constexpr int LB = R / 4;       // bytes of a row one lane loads
  constexpr int kUnroll = kUnrollBytes / LB;  // 16-token tiles per warp in flight
  static_assert(R % 32 == 0 && (LB == 8 || LB == 16), "rank");

  extern __shared__ uint32_t score_dyn[];
  uint32_t* s_key = score_dyn;                                      // [chunk]
  int32_t* s_page = reinterpret_cast<int32_t*>(score_dyn + chunk);  // [chunk / page_size + 1]
  __shared__ float s_qbar[D];
  __shared__ float s_p[R];
  __shared__ uint8_t s_dig[kDigits][R];
  __shared__ float s_scale[kDigits];
  __shared__ uint32_t s_hist[kBins];
  __shared__ uint32_t s_red[kBins];
  __shared__ uint32_t s_tot;
  __shared__ uint32_t s_warp[kWarps];
  __shared__ uint32_t s_rc[kMaxClusterCtas * kWarps];  // rank 0: candidates per region
  __shared__ uint32_t s_rgt[kMaxClusterCtas * kWarps], s_req[kMaxClusterCtas * kWarps];
  __shared__ int32_t s_info[4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int pair = blockIdx.y;
  const int b = pair / h_kv, h = pair % h_kv;
  const int G = h_q / h_kv;
  const int page_size = 1 << page_shift;
  const uint32_t crank = cluster_rank();
  const uint32_t C = cluster_size();
  const int max_len = max_pages * page_size;
  const unsigned lt = (1u << lane) - 1u;
  const int seg = warp_seg(chunk);

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
    if (crank == 0 && tid == 0) {
      count[pair] = L;
      if (cands.attend_tickets) cands.attend_tickets[pair] = 0;
    }
    return;
  }

  // ---- 1. projected group-mean query and its FP8 digits --------------------------------------
  for (int i = tid; i < kBins; i += kThreads) s_hist[i] = 0u;
  const uint16_t* qh = q + ((int64_t)b * h_q + (int64_t)h * G) * D;
  for (int i = tid; i < D; i += kThreads) {
    float acc = 0.f;
    for (int gg = 0; gg < G; ++gg) acc += bf16_to_f(qh[(int64_t)gg * D + i]);
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
  __syncthreads();
  if (warp == 0) {
    // digit c: scale 2^e_c puts the largest remaining component in [128, 256) -- inside the
    // E4M3 range -- and D_c = e4m3(remainder / 2^e_c); the remainder update is exact
    float rem[R / 32];
#pragma unroll
    for (int i = 0; i < R / 32; ++i) rem[i] = s_p[lane + 32 * i];
    for (int c = 0; c < kDigits; ++c) {
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < R / 32; ++i) m = fmaxf(m, fabsf(rem[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sc = 0.f, inv = 0.f;
      if (m > 0.f) {
        const int ex = (int)((__float_as_uint(m) >> 23) & 0xFF) - 127 - 7;
        sc = ldexpf(1.0f, ex);
        inv = ldexpf(1.0f, -ex);
      }
#pragma unroll
      for (int i = 0; i < R / 32; ++i) {
        uint8_t code = 0;
        if (m > 0.f) {
          uint16_t pk;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(pk) : "f"(rem[i] * inv));
          code = (uint8_t)(pk & 0xFF);
          rem[i] -= e4m3x2_to_f2((uint16_t)code).x * sc;
        }
        s_dig[c][lane + 32 * i] = code;
      }
      if (lane == 0) s_scale[c] = sc;
    }
  }

  // ---- 2. page list of this chunk ------------------------------------------------------------
  const int n_local = max(0, min(chunk, L - start));
  const int n_pages_local = (n_local + page_size - 1) >> page_shift;
  const int32_t* bt = block_table + (int64_t)b * max_pages + (start >> page_shift);
  for (int i = tid; i < n_pages_local; i += kThreads) {
    int32_t pg = bt[i];
    if (pg < 0 || (int64_t)pg >= num_pages) {
      raise_flag(1u);
      pg = -1;
    }
    s_page[i] = pg;
  }
  __syncthreads();
  // B fragments: column n = digit g; k-block kb, k-slot 4t+j <-> row byte t*LB + 8kb + j and
  // k-slot 16+4t+j <-> byte t*LB + 8kb + 4 + j (the same permutation is applied to the rows)
  uint32_t bd0[KB], bd1[KB];
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) {
    bd0[kb] = 0u;
    bd1[kb] = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      bd0[kb] |= (uint32_t)s_dig[g][t * LB + 8 * kb + j] << (8 * j);
      bd1[kb] |= (uint32_t)s_dig[g][t * LB + 8 * kb + 4 + j] << (8 * j);
    }
  }
  const float sc0 = s_scale[2 * t], sc1 = s_scale[2 * t + 1];

  // The scoring rows of the new token are written by the preceding store kernel.
  pdl_wait();

  // ---- 3. scores -> keys in shared memory, first-digit histogram -----------------------------
  const int n_tiles = (n_local + 15) >> 4;
  const int64_t head_off = ((int64_t)h << page_shift) * R;
  const int64_t page_bytes = ((int64_t)h_kv << page_shift) * R;
  const int pmask = page_size - 1;
  for (int t0 = warp * kUnroll; t0 < n_tiles; t0 += kWarps * kUnroll) {
    uint32_t ra[kUnroll][LB / 4], rb[kUnroll][LB / 4];  // rows g and g+8 of each tile
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int tok_a = (t0 + u) * 16 + g, tok_b = tok_a + 8;
      const int pa = tok_a < n_local ? s_page[tok_a >> page_shift] : -1;
      const int pb = tok_b < n_local ? s_page[tok_b >> page_shift] : -1;
      const uint8_t* sa = score_cache + (int64_t)pa * page_bytes + head_off +
                          (int64_t)(tok_a & pmask) * R + t * LB;
      const uint8_t* sb = score_cache + (int64_t)pb * page_bytes + head_off +
                          (int64_t)(tok_b & pmask) * R + t * LB;
      if (LB == 8) {
        const uint2 va = pa >= 0 ? ld_stream_v2(sa) : make_uint2(0u, 0u);
        const uint2 vb = pb >= 0 ? ld_stream_v2(sb) : make_uint2(0u, 0u);
        ra[u][0] = va.x; ra[u][1] = va.y;
        rb[u][0] = vb.x; rb[u][1] = vb.y;
      } else {
        const uint4 va = pa >= 0 ? ld_stream_v4(sa) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 vb = pb >= 0 ? ld_stream_v4(sb) : make_uint4(0u, 0u, 0u, 0u);
        ra[u][0] = va.x; ra[u][1] = va.y; ra[u][LB / 4 - 2] = va.z; ra[u][LB / 4 - 1] = va.w;
        rb[u][0] = vb.x; rb[u][1] = vb.y; rb[u][LB / 4 - 2] = vb.z; rb[u][LB / 4 - 1] = vb.w;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kb = 0; kb < KB; ++kb)
        mma_e4m3(c, ra[u][2 * kb], rb[u][2 * kb], ra[u][2 * kb + 1], rb[u][2 * kb + 1], bd0[kb],
                 bd1[kb]);
      float s0 = c[0] * sc0 + c[1] * sc1;  // token g   (columns 2t, 2t+1)
      float s1 = c[2] * sc0 + c[3] * sc1;  // token g+8
      s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
      s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      const int tok = (t0 + u) * 16 + g + 8 * t;  // lane t = 0 keeps token g, t = 1 token g+8
      if (t < 2 && tok < n_local) {
        const uint32_t key = score_key(t == 0 ? s0 : s1);
        s_key[tok] = key;
        atomicAdd(&s_hist[key >> 21], 1u);
      }
    }
  }

  // ---- 4. cluster rounds: threshold bin of the top 11 key bits --------------------------------
  cluster_sync();  // round 1: every histogram of the cluster is complete
  {
    const int per = kBins / (int)C;
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
  }
  cluster_sync();  // round 2: slice sums and totals are published
  if (warp == 0) {
    const int per = kBins / (int)C;
    // slice totals, top slice first: lane i holds slice C-1-i
    const uint32_t tv = (lane < (int)C) ? *remote(&s_tot, C - 1 - (uint32_t)lane) : 0u;
    const uint32_t incl = warp_incl_scan(tv, lane);
    const uint32_t excl = incl - tv;
    const unsigned hit = __ballot_sync(0xffffffffu, lane < (int)C && excl < (uint32_t)budget &&
                                                        incl >= (uint32_t)budget);
    // (always found for consistent counts; the fallback keeps every address in the cluster)
    const int sl = hit ? __ffs(hit) - 1 : 0;
    const uint32_t above_slice = __shfl_sync(0xffffffffu, excl, sl);
    const uint32_t rank_sl = C - 1 - (uint32_t)sl;
    const uint32_t* red = remote(s_red, rank_sl);
    int bin;
    uint32_t above, cnt;
    bool found;
    find_bin([&](int j) { return red[j]; }, per, above_slice, (uint32_t)budget, lane, bin, above,
             cnt, found);
    if (lane == 0) {
      if (!hit || !found) raise_flag(8u);
      s_info[0] = (int)rank_sl * per + bin;          // the threshold digit
      s_info[1] = (int)((uint32_t)budget - above);   // rank of the threshold inside its bin
      s_info[2] = (int)cnt;                          // keys in the threshold bin
    }
  }
  __syncthreads();
  const uint32_t lo_key = (uint32_t)s_info[0] << 21;  // keys below this can not be selected

  // ---- 5. every warp compacts its candidates (keys >= lo_key) in position order --------------
  {
    const int w0 = min(n_local, warp * seg), w1 = min(n_local, w0 + seg);
    const int64_t base = (int64_t)pair * C * kWarps * seg + (int64_t)(crank * kWarps + warp) * seg;
    uint32_t n_c = 0;
    for (int i0 = w0; i0 < w1; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t key = i < w1 ? s_key[i] : 0u;
      const bool c = i < w1 && key >= lo_key;
      const unsigned m = __ballot_sync(0xffffffffu, c);
      if (c) {
        const uint32_t at = n_c + __popc(m & lt);
        cands.key[base + at] = key;
        cands.pos[base + at] = start + i;
      }
      n_c += __popc(m);
    }
    if (lane == 0) cands.cnt[(int64_t)pair * kMaxClusterCtas * kWarps + crank * kWarps + warp] = n_c;
  }
  cluster_sync();  // round 3: every warp's candidates are in the workspace
  pdl_trigger();
  if (crank != 0) return;

  // ---- 6. rank 0: exact threshold among the candidates, then the ordered index set ------------
  const int n_reg = (int)C * kWarps;  // regions in position order
  for (int r = tid; r < n_reg; r += kThreads)
    s_rc[r] = cands.cnt[(int64_t)pair * kMaxClusterCtas * kWarps + r];
  uint32_t want = (uint32_t)s_info[1];
  const uint32_t in_bin = (uint32_t)s_info[2];
  uint32_t prefix = lo_key, pmask_key = 0xFFE00000u;
  uint32_t thr = 0;
  bool resolved = false;
  if (want == in_bin) {  // the whole threshold bin is selected
    thr = lo_key - 1u;   // lo_key > 0: keys of finite scores are >= 0x00800000
    want = 0;
    resolved = true;
  }
  __syncthreads();
  const uint32_t* ck = cands.key + (int64_t)pair * C * kWarps * seg;
  const int32_t* cp = cands.pos + (int64_t)pair * C * kWarps * seg;
#pragma unroll 1
  for (int pass = 1; pass <= 2 && !resolved; ++pass) {
    const int shift = pass == 1 ? 10 : 0;
    const int nb = pass == 1 ? 2048 : 1024;
    for (int i = tid; i < nb; i += kThreads) s_hist[i] = 0u;
    __syncthreads();
    for (int r = warp; r < n_reg; r += kWarps) {
      const uint32_t n = s_rc[r];
      const uint32_t* kr = ck + (int64_t)r * seg;
      for (uint32_t i = lane; i < n; i += 32) {
        const uint32_t key = kr[i];
        if ((key & pmask_key) == prefix) atomicAdd(&s_hist[(key >> shift) & (nb - 1)], 1u);
      }
    }
    __syncthreads();
    if (warp == 0) {
      int bin;
      uint32_t above, cnt;
      bool found;
      find_bin([&](int j) { return s_hist[j]; }, nb, 0u, want, lane, bin, above, cnt, found);
      if (lane == 0) {
        if (!found) raise_flag(8u);
        s_info[0] = bin;
        s_info[1] = (int)above;
        s_info[2] = (int)cnt;
      }
    }
    __syncthreads();
    want -= (uint32_t)s_info[1];
    prefix |= (uint32_t)s_info[0] << shift;
    pmask_key |= (uint32_t)(nb - 1) << shift;
    if (want == (uint32_t)s_info[2]) {
      thr = prefix - 1u;
      want = 0;
      resolved = true;
    } else if (pass == 2) {
      thr = prefix;
      resolved = true;
    }
    __syncthreads();
  }
  // per region: keys above thr, keys equal to thr
  for (int r = warp; r < n_reg; r += kWarps) {
    const uint32_t n = s_rc[r];
    const uint32_t* kr = ck + (int64_t)r * seg;
    uint32_t n_gt = 0, n_eq = 0;
    for (uint32_t i0 = 0; i0 < n; i0 += 32) {
      const uint32_t i = i0 + lane;
      const uint32_t key = i < n ? kr[i] : 0u;
      n_gt += __popc(__ballot_sync(0xffffffffu, i < n && key > thr));
      n_eq += __popc(__ballot_sync(0xffffffffu, i < n && key == thr));
    }
    if (lane == 0) {
      s_rgt[r] = n_gt;
      s_req[r] = n_eq;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive prefixes over regions (in position order) of equal keys and of selected keys;
    // s_rgt becomes the region's output offset, s_req the number of equal keys seen before it
    constexpr int kPer = kMaxClusterCtas * kWarps / 32;
    uint32_t gt[kPer], eq[kPer], se = 0, ss = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int r = lane * kPer + i;
      gt[i] = r < n_reg ? s_rgt[r] : 0u;
      eq[i] = r < n_reg ? s_req[r] : 0u;
      se += eq[i];
    }
    const uint32_t eq_before_lane = warp_incl_scan(se, lane) - se;
    uint32_t e = eq_before_lane;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const uint32_t rem = want > e ? want - e : 0u;
      const uint32_t tk = eq[i] < rem ? eq[i] : rem;
      ss += gt[i] + tk;
      e += eq[i];
    }
    const uint32_t sel_before_lane = warp_incl_scan(ss, lane) - ss;
    e = eq_before_lane;
    uint32_t o = sel_before_lane;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int r = lane * kPer + i;
      const uint32_t rem = want > e ? want - e : 0u;
      const uint32_t tk = eq[i] < rem ? eq[i] : rem;
      if (r < n_reg) {
        s_rgt[r] = o;
        s_req[r] = e;
      }
      o += gt[i] + tk;
      e += eq[i];
    }
    if (lane == 31 && o != (uint32_t)budget) raise_flag(8u);
  }
  __syncthreads();
  for (int r = warp; r < n_reg; r += kWarps) {
    const uint32_t n = s_rc[r];
    const uint32_t* kr = ck + (int64_t)r * seg;
    const int32_t* pr = cp + (int64_t)r * seg;
    uint32_t pos = s_rgt[r], eqs = s_req[r];
    for (uint32_t i0 = 0; i0 < n; i0 += 32) {
      const uint32_t i = i0 + lane;
      const uint32_t key = i < n ? kr[i] : 0u;
      const bool is_eq = i < n && key == thr;
      const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
      const bool take = (i < n && key > thr) || (is_eq && eqs + __popc(eqm & lt) < want);
      const unsigned selm = __ballot_sync(0xffffffffu, take);
      const uint32_t at = pos + __popc(selm & lt);
      if (take && at < (uint32_t)budget) out_idx[at] = pr[i];
      pos += __popc(selm);
      eqs += __popc(eqm);
    }
  }
  if (tid == 0) {
    count[pair] = budget;
    // the attention launched next merges its splits through these counters
    if (cands.attend_tickets) cands.attend_tickets[pair] = 0;
  }
}

template <int D, int R>
cudaError_t launch_t(const ScorePlan& plan, int pairs, bool pdl, cudaStream_t s, const uint16_t* q,
                     const float* basis, const uint8_t* score_cache, const int32_t* block_table,
                     int max_pages, const int32_t* seq_lens, int h_q, int h_kv, int64_t num_pages,
                     int page_shift, int budget, int32_t* idx, int32_t* count, void* ws,
                     int* attend_tickets) {
  auto kern = score_topk_kernel<D, R>;
  cudaError_t e = configure_kernel((const void*)kern, (int)plan.smem, plan.cluster > 8);
  if (e != cudaSuccess) return e;
  Cands cands;
  uint8_t* w = static_cast<uint8_t*>(ws);
  cands.cnt = reinterpret_cast<uint32_t*>(w);
  const size_t n_entries = (size_t)pairs * plan.cluster * kWarps * warp_seg(plan.chunk);
  cands.key = reinterpret_cast<uint32_t*>(w + cand_bytes_counts(pairs));
  cands.pos = reinterpret_cast<int32_t*>(w + cand_bytes_counts(pairs) + n_entries * 4);
  cands.attend_tickets = attend_tickets;
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
                         h_kv, num_pages, page_shift, budget, plan.chunk, idx, count, cands);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace score_detail

ScorePlan plan_score(int pairs, int max_seq_len, int page_size) {
  ScorePlan p;
  // tokens per CTA: a multiple of the page size (a CTA's pages start on a page) and of 256
  // (whole 16-token tiles for every warp)
  int align = 256;
  while (align % page_size) align *= 2;
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
  p.ws_bytes = score_detail::cand_bytes_counts(pairs) +
               (size_t)pairs * c * score_detail::kWarps * score_detail::warp_seg(chunk) * 8;
  return p;
}

cudaError_t launch_score_topk(const uint16_t* q, const float* basis, const uint8_t* score_cache,
                              const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                              int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                              int page_size, int budget, int32_t* idx, int32_t* count, void* ws,
                              int* attend_tickets, bool pdl, cudaStream_t s) {
  const int pairs = batch * h_kv;
  if (pairs == 0) return cudaSuccess;
  const ScorePlan plan = plan_score(pairs, max_pages * page_size, page_size);
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  if (d == 128 && r == 32)
    return score_detail::launch_t<128, 32>(plan, pairs, pdl, s, q, basis, score_cache, block_table,
                                           max_pages, seq_lens, h_q, h_kv, num_pages, shift,
                                           budget, idx, count, ws, attend_tickets);
  if (d == 128 && r == 64)
    return score_detail::launch_t<128, 64>(plan, pairs, pdl, s, q, basis, score_cache, block_table,
                                           max_pages, seq_lens, h_q, h_kv, num_pages, shift,
                                           budget, idx, count, ws, attend_tickets);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
