// Score + top-B (JSSA summary, eq. (1) and section 3.1 steps 1-2; JSSA README, section 4:
// jssa_budget tokens per decode step and KV head). Three kernels, chained on one stream with
// programmatic dependent launch:
//
// prep   one CTA per (sequence, KV head). p = M_h qbar (qbar = mean of the G query heads of KV
//        head h), fp32, written as a sum of 8 FP8 "digit" vectors with power-of-two column
//        scales, p = sum_c 2^e_c D_c with D_c in E4M3 (digit c rounds what the earlier digits
//        left), which represents p to ~2^-32 of its largest component. Then a candidate
//        threshold: the scores of a stratified random sample of 2048 positions give a key that
//        about twice the budget (plus a margin of several standard deviations) of all tokens
//        reach. The threshold only decides how many keys travel to the select kernel -- the
//        selection itself is exact (see select). At decode the same kernel first stores the new
//        token: its K and V rows and its scoring code e4m3(M_h k) (float64 sum, one rounding).
// scan   CTAs over (chunk of positions, sequence x KV head), no cluster and no shared key array:
//        a pure stream of the FP8 scoring rows (page-table indexed, 8-byte non-allocating loads,
//        register double buffering). The codes are consumed as they are by the tensor cores: one
//        mma.sync m16n8k32 E4M3 x E4M3 -> fp32 per 16 tokens and 32 code bytes multiplies the 16
//        rows by the 8 digit columns, and s = sum_c 2^e_c C[:, c]. (Widening the codes on the
//        CUDA cores costs ~3 instructions per byte and leaves this HBM-bound loop issue-bound.)
//        Every warp walks a contiguous run of tiles and appends the keys at or above the
//        threshold, with their positions, to its own workspace region in position order.
// select one CTA per (sequence, KV head): the exact budget-th largest key among the candidates
//        (radix digits of 11, 11 and 10 bits over order-preserving 32-bit keys), every key above
//        it and the equal keys in position order up to the budget (ties go to the lower
//        position), written as the index set in ascending order. If the candidates are fewer
//        than the budget (the sampled threshold was too high -- not expected in practice), the
//        CTA first rescans the sequence with no threshold, so the result is exact in every case.
// seq_len <= budget selects every position without scoring.
#include "common.cuh"

namespace jssa {

namespace score_detail {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnrollBytes = 32;   // bytes of scoring rows per lane per load batch
constexpr int kBins = 2048;
constexpr int kDigits = 8;         // FP8 digit columns of p (the n = 8 of the mma)
constexpr int kSample = 2048;      // sampled positions per (sequence, KV head)
constexpr int kExactMax = 16384;   // up to this context every token is a candidate
constexpr int kSelectCap = 16384;  // candidates the select kernel stages in shared memory
constexpr int kMaxRegions = 4096;  // scan regions (chunks x warps) per (sequence, KV head)
constexpr int kPrepBytes = 1024;   // per (sequence, KV head): digits, scales, threshold, mode
constexpr int kPrepScale = 512, kPrepThr = 544, kPrepMode = 548;
constexpr int kModeScan = 0, kModeAll = 1;

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

// Bin of a histogram (`nb` bins, read through `at`) holding the want-th largest element counted
// from the top. Warp-wide; returns (bin, count of elements in strictly higher bins, count in
// the bin) on every lane.
template <typename At>
__device__ __forceinline__ void find_bin(At at, int nb, uint32_t want, int lane, int& bin_out,
                                         uint32_t& above_out, uint32_t& cnt_out, bool& found) {
  const int bpl = (nb + 31) / 32;
  const int hi = nb - lane * bpl;
  const int lo = max(0, hi - bpl);
  uint32_t c = 0;
  for (int j = lo; j < hi; ++j) c += at(j);
  const uint32_t incl = warp_incl_scan(c, lane);
  const uint32_t excl = incl - c;
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

// Exact radix select over `n` keys read through `key_at(i)`: the threshold key thr and the number
// `take` of keys equal to thr that belong to the want largest (ties are resolved afterwards by
// position); every key > thr belongs to them. Block-wide; uses s_hist[kBins] and s_info[3].
template <typename KeyAt>
__device__ void radix_select(KeyAt key_at, int n, uint32_t want, uint32_t* s_hist, int* s_info,
                             uint32_t& thr, uint32_t& take) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, pmask = 0;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    for (int i = tid; i < nb; i += kThreads) s_hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t key = key_at(i);
      if ((key & pmask) == prefix) atomicAdd(&s_hist[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      int bin;
      uint32_t above, cnt;
      bool found;
      find_bin([&](int j) { return s_hist[j]; }, nb, want, lane, bin, above, cnt, found);
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
    pmask |= (uint32_t)(nb - 1) << shift;
    const uint32_t in_bin = (uint32_t)s_info[2];
    __syncthreads();
    if (want == in_bin) {  // the whole bin is taken: everything >= its lowest key
      thr = prefix - 1u;   // prefix > 0: keys of finite scores are >= 0x00800000
      take = 0;
      return;
    }
  }
  thr = prefix;
  take = want;
}

struct Prep {
  uint8_t* rec;  // [pairs][kPrepBytes]: digits [8][R] at 0, scales at kPrepScale, threshold
                 // key at kPrepThr, mode at kPrepMode
};
struct Cands {
  uint32_t* key;       // [pairs][n_chunks][kWarps][chunk / kWarps]
  int32_t* pos;        // same layout
  uint32_t* cnt;       // [pairs][n_chunks][kWarps]
  int* attend_tickets; // [pairs] split-K tickets of the attention that follows, or null
};

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}

// Fragment registers of the digit matrix (B operand): column n = digit g; k-block kb, k-slot
// 4t+j <-> row byte t*LB + 8kb + j and k-slot 16+4t+j <-> byte t*LB + 8kb + 4 + j (the same
// permutation is applied to the code rows, so the dot products are unchanged).
template <int R>
struct DigitFrags {
  uint32_t b0[R / 32], b1[R / 32];
  float sc0, sc1;
  __device__ __forceinline__ void load(const uint8_t* dig, const float* scale, int lane) {
    constexpr int LB = R / 4;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kb = 0; kb < R / 32; ++kb) {
      b0[kb] = 0u;
      b1[kb] = 0u;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b0[kb] |= (uint32_t)dig[g * R + t * LB + 8 * kb + j] << (8 * j);
        b1[kb] |= (uint32_t)dig[g * R + t * LB + 8 * kb + 4 + j] << (8 * j);
      }
    }
    sc0 = scale[2 * t];
    sc1 = scale[2 * t + 1];
  }
};

// Scores of a 16-token tile: ra / rb are the permuted code rows of tokens g and g+8 held by lane
// (g, t); on return every lane of the quad has token g's score in s0 and token g+8's in s1.
template <int R>
__device__ __forceinline__ void tile_scores(const uint32_t* ra, const uint32_t* rb,
                                            const DigitFrags<R>& df, float& s0, float& s1) {
  float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kb = 0; kb < R / 32; ++kb)
    mma_e4m3(c, ra[2 * kb], rb[2 * kb], ra[2 * kb + 1], rb[2 * kb + 1], df.b0[kb], df.b1[kb]);
  s0 = c[0] * df.sc0 + c[1] * df.sc1;  // token g   (columns 2t, 2t+1)
  s1 = c[2] * df.sc0 + c[3] * df.sc1;  // token g+8
  s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
  s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
  s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
  s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
}

template <int R>
__device__ __forceinline__ void load_row(uint32_t* dst, const uint8_t* src, bool ok) {
  if (R == 32) {
    const uint2 v = ok ? ld_stream_v2(src) : make_uint2(0u, 0u);
    dst[0] = v.x;
    dst[1] = v.y;
  } else {
    const uint4 v = ok ? ld_stream_v4(src) : make_uint4(0u, 0u, 0u, 0u);
    dst[0] = v.x;
    dst[1] = v.y;
    dst[2] = v.z;
    dst[3] = v.w;
  }
}

// ------------------------------------------------------------------------------------------------
// scan of one chunk; the body is shared with the select kernel's rescue path
// ------------------------------------------------------------------------------------------------

struct ScanArgs {
  const uint8_t* score_cache;
  const int32_t* block_table;
  int max_pages;
  const int32_t* seq_lens;
  int h_kv;
  int64_t num_pages;
  int page_shift;
  int chunk;      // positions per scan CTA (multiple of 128 and of the page size)
  int n_chunks;   // chunks per (sequence, KV head)
  int budget;
  Prep prep;
  Cands cands;
};

struct ChunkGeom {
  const uint8_t* head_base;  // scoring cache + this head's offset inside a page
  uint32_t page_bytes;       // bytes of one page (all heads)
  int page_shift;
  int n_local;               // valid tokens in this chunk
  int start;                 // first position of the chunk
};

template <int R>
struct ScanBuf {
  static constexpr int kUnroll = kUnrollBytes / (R / 4);
  uint32_t ra[kUnroll][R / 16], rb[kUnroll][R / 16];
};

template <int R>
__device__ __forceinline__ void scan_load(ScanBuf<R>& buf, const ChunkGeom& cg,
                                          const int32_t* s_page, int t0, int t_end, int lane) {
  constexpr int LB = R / 4;
  const int g = lane >> 2, t = lane & 3;
  const int pmask = (1 << cg.page_shift) - 1;
#pragma unroll
  for (int u = 0; u < ScanBuf<R>::kUnroll; ++u) {
    const bool live = t0 + u < t_end;
    const int ta = (t0 + u) * 16 + g, tb = ta + 8;
    // (a 16-token tile crosses pages only when the page size is below 16)
    const int pa = live && ta < cg.n_local ? s_page[ta >> cg.page_shift] : -1;
    const int pb = live && tb < cg.n_local ? s_page[tb >> cg.page_shift] : -1;
    load_row<R>(buf.ra[u], cg.head_base + (int64_t)pa * cg.page_bytes + (ta & pmask) * R + t * LB,
                pa >= 0);
    load_row<R>(buf.rb[u], cg.head_base + (int64_t)pb * cg.page_bytes + (tb & pmask) * R + t * LB,
                pb >= 0);
  }
}

// Keys >= thr of tiles [t0, t0 + kUnroll) appended in position order to this warp's region.
template <int R>
__device__ __forceinline__ void scan_emit(const ScanBuf<R>& buf, const DigitFrags<R>& df,
                                          const ChunkGeom& cg, int t0, int t_end, uint32_t thr,
                                          uint32_t* rkey, int32_t* rpos, uint32_t& run, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int u = 0; u < ScanBuf<R>::kUnroll; ++u) {
    float s0, s1;
    tile_scores<R>(buf.ra[u], buf.rb[u], df, s0, s1);
    const int tok = (t0 + u) * 16 + g + 8 * t;  // lane t = 0 keeps token g, t = 1 token g+8
    const uint32_t key = score_key(t == 0 ? s0 : s1);
    const bool c = t < 2 && t0 + u < t_end && tok < cg.n_local && key >= thr;
    const unsigned m = __ballot_sync(0xffffffffu, c);
    // position order inside the tile: tokens 0..7 sit on lanes 4g (t = 0), 8..15 on 4g+1
    const unsigned m0 = m & 0x11111111u, m1 = m & 0x22222222u;
    if (c) {
      const uint32_t at = run + (t == 0 ? __popc(m0 & lt) : __popc(m0) + __popc(m1 & lt));
      rkey[at] = key;
      rpos[at] = cg.start + tok;
    }
    run += __popc(m);
  }
}

// One warp's contiguous run of tiles [t_begin, t_end), register double-buffered.
template <int R>
__device__ __forceinline__ uint32_t scan_warp(const ChunkGeom& cg, const int32_t* s_page,
                                              const DigitFrags<R>& df, uint32_t thr, int t_begin,
                                              int t_end, uint32_t* rkey, int32_t* rpos, int lane) {
  constexpr int kU = ScanBuf<R>::kUnroll;
  uint32_t run = 0;
  ScanBuf<R> a, b;
  int t0 = t_begin;
  if (t0 < t_end) scan_load<R>(a, cg, s_page, t0, t_end, lane);
  while (t0 < t_end) {
    if (t0 + kU < t_end) scan_load<R>(b, cg, s_page, t0 + kU, t_end, lane);
    scan_emit<R>(a, df, cg, t0, t_end, thr, rkey, rpos, run, lane);
    t0 += kU;
    if (t0 >= t_end) break;
    if (t0 + kU < t_end) scan_load<R>(a, cg, s_page, t0 + kU, t_end, lane);
    scan_emit<R>(b, df, cg, t0, t_end, thr, rkey, rpos, run, lane);
    t0 += kU;
  }
  return run;
}

// Page list of a chunk into shared memory (bounds checked; -1 = unusable page).
__device__ __forceinline__ void load_pages(int32_t* s_page, const int32_t* bt, int n_pages,
                                           int64_t num_pages) {
  for (int i = threadIdx.x; i < n_pages; i += kThreads) {
    int32_t pg = bt[i];
    if (pg < 0 || (int64_t)pg >= num_pages) {
      raise_flag(1u);
      pg = -1;
    }
    s_page[i] = pg;
  }
}

__device__ __forceinline__ int clamp_len(int L, int max_len) {
  if (L < 0 || L > max_len) {
    if (threadIdx.x == 0) raise_flag(4u);
    return L < 0 ? 0 : max_len;
  }
  return L;
}

// Scan of chunk c of pair `pair` by the calling CTA (page list already in s_page); writes this
// chunk's kWarps regions and their counts.
template <int R>
__device__ void scan_chunk(const ScanArgs& a, int pair, int c, int L, uint32_t thr,
                           const DigitFrags<R>& df, const int32_t* s_page) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = pair % a.h_kv;
  ChunkGeom cg;
  cg.start = c * a.chunk;
  cg.n_local = max(0, min(a.chunk, L - cg.start));
  cg.page_shift = a.page_shift;
  cg.page_bytes = ((uint32_t)a.h_kv << a.page_shift) * R;
  cg.head_base = a.score_cache + ((int64_t)h << a.page_shift) * R;
  const int seg = a.chunk / kWarps;
  const int64_t region = (((int64_t)pair * a.n_chunks + c) * kWarps + warp) * seg;
  const int n_tiles = (cg.n_local + 15) >> 4;
  const int tpw = seg / 16;  // tiles per warp (one region)
  const int t_begin = min(n_tiles, warp * tpw), t_end = min(n_tiles, t_begin + tpw);
  const uint32_t n = scan_warp<R>(cg, s_page, df, thr, t_begin, t_end, a.cands.key + region,
                                  a.cands.pos + region, lane);
  if (lane == 0) a.cands.cnt[((int64_t)pair * a.n_chunks + c) * kWarps + warp] = n;
}

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 3) scan_kernel(ScanArgs a) {
  extern __shared__ int32_t scan_pages[];  // chunk / page_size + 1 entries
  const int c = blockIdx.x, pair = blockIdx.y;
  const int b = pair / a.h_kv;
  const int L = clamp_len(a.seq_lens[b], a.max_pages << a.page_shift);
  const int start = c * a.chunk;
  const int n_local = max(0, min(a.chunk, L - start));
  const int n_pages = (n_local + (1 << a.page_shift) - 1) >> a.page_shift;
  load_pages(scan_pages, a.block_table + (int64_t)b * a.max_pages + (start >> a.page_shift),
             n_pages, a.num_pages);
  __syncthreads();
  pdl_wait();  // digits, threshold and the new token's code come from the prep kernel
  const uint8_t* rec = a.prep.rec + (int64_t)pair * kPrepBytes;
  const int mode = *reinterpret_cast<const int*>(rec + kPrepMode);
  if (mode == kModeAll || n_local == 0) {
    if ((threadIdx.x & 31) == 0)
      a.cands.cnt[((int64_t)pair * a.n_chunks + c) * kWarps + (threadIdx.x >> 5)] = 0u;
    pdl_trigger();
    return;
  }
  DigitFrags<R> df;
  df.load(rec, reinterpret_cast<const float*>(rec + kPrepScale), threadIdx.x & 31);
  const uint32_t thr = *reinterpret_cast<const uint32_t*>(rec + kPrepThr);
  scan_chunk<R>(a, pair, c, L, thr, df, scan_pages);
  pdl_trigger();
}

// ------------------------------------------------------------------------------------------------
// prep
// ------------------------------------------------------------------------------------------------

struct PrepArgs {
  const uint16_t* q;
  const float* basis;
  const uint8_t* score_cache;
  const int32_t* block_table;
  int max_pages;
  const int32_t* seq_lens;
  int h_q, h_kv;
  int64_t num_pages;
  int page_shift;
  int budget;
  Prep prep;
  StoreNew store;  // decode: the new token (position seq_len - 1)
};

template <int D, int R, bool STORE>
__global__ void __launch_bounds__(kThreads) prep_kernel(PrepArgs a) {
  constexpr int LB = R / 4;
  __shared__ float s_qbar[D];
  __shared__ float s_p[R];
  __shared__ float s_k[D];
  __shared__ __align__(16) uint8_t s_dig[kDigits * R];
  __shared__ float s_scale[kDigits];
  __shared__ uint32_t s_skey[kSample];
  __shared__ int64_t s_srow[kSample];
  __shared__ uint32_t s_hist[kBins];
  __shared__ int s_info[4];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = blockIdx.x;
  const int b = pair / a.h_kv, h = pair % a.h_kv;
  const int G = a.h_q / a.h_kv;
  const int page_size = 1 << a.page_shift;
  const int L = clamp_len(a.seq_lens[b], a.max_pages << a.page_shift);
  const int32_t* bt = a.block_table + (int64_t)b * a.max_pages;
  const float* m_h = a.basis + (int64_t)h * R * D;

  // ---- decode: store the new token (K/V rows and scoring code) ---------------------------------
  if (STORE && L > 0) {
    const StoreNew& st = a.store;
    const int pos = L - 1;
    const int32_t page = bt[pos >> a.page_shift];
    const int off = pos & (page_size - 1);
    const bool ok = page >= 0 && (int64_t)page < a.num_pages;
    if (!ok && tid == 0) raise_flag(1u);
    const uint16_t* krow = st.k_new + ((int64_t)b * a.h_kv + h) * D;
    const uint16_t* vrow = st.v_new + ((int64_t)b * a.h_kv + h) * D;
    for (int i = tid; i < D; i += kThreads) s_k[i] = bf16_to_f(krow[i]);
    if (ok) {
      const int64_t base = (int64_t)page * st.page_stride + (int64_t)off * st.slot_stride +
                           (int64_t)h * st.head_stride;
      for (int i = tid; i < D; i += kThreads) {
        st.k_cache[base + i] = krow[i];
        st.v_cache[base + i] = vrow[i];
      }
    }
    __syncthreads();
    if (ok) {
      uint8_t* dst = st.score_cache + (((int64_t)page * a.h_kv + h) * page_size + off) * R;
      for (int j = tid; j < R; j += kThreads) {
        const float* mrow = m_h + (int64_t)j * D;
        double acc = 0.0;
        for (int i = 0; i < D; ++i) acc = fma((double)mrow[i], (double)s_k[i], acc);
        dst[j] = f64_to_e4m3(acc);
      }
    }
  }

  // ---- projected group-mean query and its FP8 digits -------------------------------------------
  const uint16_t* qh = a.q + ((int64_t)b * a.h_q + (int64_t)h * G) * D;
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
    const float* mrow = m_h + (int64_t)j * D + sub * DPT;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < DPT; ++i) acc = fmaf(mrow[i], s_qbar[sub * DPT + i], acc);
#pragma unroll
    for (int o = TPJ / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (sub == 0) s_p[j] = acc;
  }
  __syncthreads();
  if (warp == 0) {
    // digit c: the scale 2^e_c puts the largest remaining component in [128, 256), inside the
    // E4M3 range, and D_c = e4m3(remainder / 2^e_c); the remainder update is exact
    float rem[R / 32];
#pragma unroll
    for (int i = 0; i < R / 32; ++i) rem[i] = s_p[lane + 32 * i];
    for (int c = 0; c < kDigits; ++c) {
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < R / 32; ++i) mx = fmaxf(mx, fabsf(rem[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sc = 0.f, inv = 0.f;
      if (mx > 0.f) {
        const int ex = (int)((__float_as_uint(mx) >> 23) & 0xFF) - 127 - 7;
        sc = ldexpf(1.0f, ex);
        inv = ldexpf(1.0f, -ex);
      }
#pragma unroll
      for (int i = 0; i < R / 32; ++i) {
        uint8_t code = 0;
        if (mx > 0.f) {
          uint16_t pk;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(pk) : "f"(rem[i] * inv));
          code = (uint8_t)(pk & 0xFF);
          rem[i] -= e4m3x2_to_f2((uint16_t)code).x * sc;
        }
        s_dig[c * R + lane + 32 * i] = code;
      }
      if (lane == 0) s_scale[c] = sc;
    }
  }
  __syncthreads();
  uint8_t* rec = a.prep.rec + (int64_t)pair * kPrepBytes;
  for (int i = tid; i < kDigits * R; i += kThreads) rec[i] = s_dig[i];
  if (tid < kDigits) reinterpret_cast<float*>(rec + kPrepScale)[tid] = s_scale[tid];

  // ---- candidate threshold --------------------------------------------------------------------
  int mode = kModeScan;
  uint32_t thr = 0u;  // every key of a finite score is above 0
  if (L <= a.budget) {
    mode = kModeAll;
  } else if (L > kExactMax) {
    const double expect = (double)a.budget * kSample / (double)L;
    const int k = (int)ceil(2.0 * expect + 4.0 * sqrt(expect) + 8.0);
    if (k < kSample / 2) {
      // stratified sample: one position per stratum of L / kSample tokens (never the new
      // token, whose code this kernel may have just written)
      const int stratum = L / kSample;
      for (int i = tid; i < kSample; i += kThreads) {
        const uint32_t hsh = mix32((uint32_t)i * 0x9E3779B9u ^ ((uint32_t)pair * 0x85EBCA6Bu + 1u));
        int pos = i * stratum + (int)(hsh % (uint32_t)stratum);
        if (pos >= L - 1) pos = L - 2;
        const int32_t pg = bt[pos >> a.page_shift];
        s_srow[i] = (pg < 0 || (int64_t)pg >= a.num_pages)
                        ? (int64_t)-1
                        : (((int64_t)pg * a.h_kv + h) << a.page_shift) + (pos & (page_size - 1));
      }
      __syncthreads();
      DigitFrags<R> df;
      df.load(s_dig, s_scale, lane);
      const int g = lane >> 2, t = lane & 3;
      // 128 tiles of 16 samples, 16 per warp in two batches of 8; loads issued before the math
      constexpr int kBatch = 8;
      for (int bt0 = 0; bt0 < kSample / 16 / kWarps; bt0 += kBatch) {
        uint32_t ra[kBatch][R / 16], rb[kBatch][R / 16];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int tile = warp * (kSample / 16 / kWarps) + bt0 + u;
          const int64_t sa = s_srow[tile * 16 + g], sb = s_srow[tile * 16 + g + 8];
          load_row<R>(ra[u], a.score_cache + (sa < 0 ? 0 : sa) * R + t * LB, sa >= 0);
          load_row<R>(rb[u], a.score_cache + (sb < 0 ? 0 : sb) * R + t * LB, sb >= 0);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          float s0, s1;
          tile_scores<R>(ra[u], rb[u], df, s0, s1);
          const int tile = warp * (kSample / 16 / kWarps) + bt0 + u;
          if (t < 2) s_skey[tile * 16 + g + 8 * t] = score_key(t == 0 ? s0 : s1);
        }
      }
      __syncthreads();
      uint32_t take;
      radix_select([&](int i) { return s_skey[i]; }, kSample, (uint32_t)k, s_hist, s_info, thr,
                   take);
      // candidates: keys >= the k-th largest sampled key (radix_select returns that key itself,
      // or one below the lowest key of a bin taken whole)
      if (take == 0u) thr += 1u;
    }
  }
  if (tid == 0) {
    *reinterpret_cast<uint32_t*>(rec + kPrepThr) = thr;
    *reinterpret_cast<int*>(rec + kPrepMode) = mode;
  }
  // complete only after the kernel before this one: the scan reads what both wrote
  pdl_wait();
  pdl_trigger();
}

// ------------------------------------------------------------------------------------------------
// select
// ------------------------------------------------------------------------------------------------

struct SelectArgs {
  ScanArgs scan;
  int32_t* idx;
  int32_t* count;
};

template <int D, int R>
__global__ void __launch_bounds__(kThreads) select_kernel(SelectArgs s) {
  extern __shared__ uint32_t sel_dyn[];  // keys [kSelectCap] then positions [kSelectCap]
  uint32_t* s_ckey = sel_dyn;
  int32_t* s_cpos = reinterpret_cast<int32_t*>(sel_dyn + kSelectCap);
  __shared__ uint32_t s_hist[kBins];
  __shared__ int s_info[4];
  __shared__ uint32_t s_roff[kMaxRegions + 1];
  __shared__ uint32_t s_wa[kWarps], s_wb[kWarps];

  const ScanArgs& a = s.scan;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = blockIdx.x;
  const int b = pair / a.h_kv;
  const int L = clamp_len(a.seq_lens[b], a.max_pages << a.page_shift);
  const int budget = a.budget;
  int32_t* out_idx = s.idx + (int64_t)pair * budget;
  const unsigned lt = (1u << lane) - 1u;
  pdl_wait();  // the scan's candidates
  const uint8_t* rec = a.prep.rec + (int64_t)pair * kPrepBytes;
  const int mode = *reinterpret_cast<const int*>(rec + kPrepMode);
  if (mode == kModeAll) {
    for (int j = tid; j < budget; j += kThreads) out_idx[j] = j < L ? j : -1;
    if (tid == 0) {
      s.count[pair] = L;
      if (a.cands.attend_tickets) a.cands.attend_tickets[pair] = 0;
    }
    pdl_trigger();
    return;
  }
  const int n_reg = a.n_chunks * kWarps;
  const int seg = a.chunk / kWarps;
  const uint32_t* ck = a.cands.key + (int64_t)pair * n_reg * seg;
  const int32_t* cp = a.cands.pos + (int64_t)pair * n_reg * seg;
  const uint32_t* cc = a.cands.cnt + (int64_t)pair * n_reg;
  const uint32_t want = (uint32_t)min(budget, L);

  // region offsets: exclusive prefix of the counts, in position order
  auto offsets = [&]() {
    if (warp == 0) {
      uint32_t run = 0;
      for (int r0 = 0; r0 < n_reg; r0 += 32) {
        const int r = r0 + lane;
        const uint32_t v = r < n_reg ? cc[r] : 0u;
        const uint32_t incl = warp_incl_scan(v, lane);
        if (r < n_reg) s_roff[r] = run + incl - v;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) s_roff[n_reg] = run;
    }
    __syncthreads();
  };
  offsets();
  if (s_roff[n_reg] < want) {
    // rescue: the sampled threshold was too high; score every token of the sequence again with
    // no threshold (all keys become candidates), then select exactly as usual
    if (tid == 0) raise_flag(16u);
    DigitFrags<R> df;
    df.load(rec, reinterpret_cast<const float*>(rec + kPrepScale), lane);
    int32_t* s_page = reinterpret_cast<int32_t*>(s_ckey);  // free until the staging below
    for (int c = 0; c < a.n_chunks; ++c) {
      const int start = c * a.chunk;
      const int n_local = max(0, min(a.chunk, L - start));
      const int n_pages = (n_local + (1 << a.page_shift) - 1) >> a.page_shift;
      __syncthreads();
      load_pages(s_page, a.block_table + (int64_t)b * a.max_pages + (start >> a.page_shift),
                 n_pages, a.num_pages);
      __syncthreads();
      scan_chunk<R>(a, pair, c, L, 0u, df, s_page);
    }
    __syncthreads();
    offsets();
  }
  const uint32_t n = s_roff[n_reg];
  const bool staged = n <= (uint32_t)kSelectCap;
  if (staged) {
    // flatten the regions into shared memory (keys and positions, position order)
    for (int r = warp; r < n_reg; r += kWarps) {
      const uint32_t cnt = s_roff[r + 1] - s_roff[r], off = s_roff[r];
      for (uint32_t i = lane; i < cnt; i += 32) {
        s_ckey[off + i] = ck[(int64_t)r * seg + i];
        s_cpos[off + i] = cp[(int64_t)r * seg + i];
      }
    }
    __syncthreads();
  }
  // flattened candidate j -> region (the last r with s_roff[r] <= j) when not staged
  auto region_of = [&](int j) {
    int lo = 0, hi = n_reg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_roff[mid] <= (uint32_t)j) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  auto key_at = [&](int j) -> uint32_t {
    if (staged) return s_ckey[j];
    const int r = region_of(j);
    return ck[(int64_t)r * seg + (j - (int)s_roff[r])];
  };
  auto pos_at = [&](int j) -> int32_t {
    if (staged) return s_cpos[j];
    const int r = region_of(j);
    return cp[(int64_t)r * seg + (j - (int)s_roff[r])];
  };
  uint32_t thr, take;
  radix_select(key_at, (int)n, want, s_hist, s_info, thr, take);
  // ordered emission: keys > thr, and the first `take` keys == thr in position order
  constexpr int kBlk = kThreads * 8;  // candidates per block, 256 per warp
  uint32_t written = 0, eq_seen = 0;
  for (uint32_t b0 = 0; b0 < n; b0 += kBlk) {
    const uint32_t w0 = min(n, b0 + (uint32_t)warp * 256u), w1 = min(n, w0 + 256u);
    uint32_t n_gt = 0, n_eq = 0;
    for (uint32_t i0 = w0; i0 < w1; i0 += 32) {
      const uint32_t i = i0 + lane;
      const uint32_t key = i < w1 ? key_at((int)i) : 0u;
      n_gt += __popc(__ballot_sync(0xffffffffu, i < w1 && key > thr));
      n_eq += __popc(__ballot_sync(0xffffffffu, i < w1 && key == thr));
    }
    if (lane == 0) {
      s_wa[warp] = n_gt;
      s_wb[warp] = n_eq;
    }
    __syncthreads();
    uint32_t eq_before = eq_seen, sel_before = written, blk_sel = 0, blk_eq = 0;
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t e_before = eq_seen + blk_eq;
      const uint32_t rem = take > e_before ? take - e_before : 0u;
      const uint32_t tk = s_wb[w] < rem ? s_wb[w] : rem;
      if (w < warp) {
        sel_before += s_wa[w] + tk;
        eq_before += s_wb[w];
      }
      blk_sel += s_wa[w] + tk;
      blk_eq += s_wb[w];
    }
    uint32_t pos = sel_before, eqs = eq_before;
    for (uint32_t i0 = w0; i0 < w1; i0 += 32) {
      const uint32_t i = i0 + lane;
      const uint32_t key = i < w1 ? key_at((int)i) : 0u;
      const bool is_eq = i < w1 && key == thr;
      const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
      const bool tk = (i < w1 && key > thr) || (is_eq && eqs + __popc(eqm & lt) < take);
      const unsigned selm = __ballot_sync(0xffffffffu, tk);
      const uint32_t at = pos + __popc(selm & lt);
      if (tk && at < (uint32_t)budget) out_idx[at] = pos_at((int)i);
      pos += __popc(selm);
      eqs += __popc(eqm);
    }
    written += blk_sel;
    eq_seen += blk_eq;
    __syncthreads();
  }
  for (int j = (int)want + tid; j < budget; j += kThreads) out_idx[j] = -1;
  if (tid == 0) {
    if (written != want) raise_flag(8u);
    s.count[pair] = (int)want;
    // the attention launched next merges its splits through these counters
    if (a.cands.attend_tickets) a.cands.attend_tickets[pair] = 0;
  }
  pdl_trigger();
}

template <typename Kern, typename Arg>
cudaError_t launch_k(Kern kern, dim3 grid, size_t smem, bool pdl, cudaStream_t s, const Arg& arg) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, arg);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int R>
cudaError_t launch_t(const ScorePlan& plan, int pairs, const PrepArgs& pa, const ScanArgs& sa,
                     const SelectArgs& sel, bool store, bool pdl, cudaStream_t s) {
  cudaError_t e;
  if (store) e = launch_k(prep_kernel<D, R, true>, dim3(pairs), 0, pdl, s, pa);
  else e = launch_k(prep_kernel<D, R, false>, dim3(pairs), 0, pdl, s, pa);
  if (e != cudaSuccess) return e;
  const size_t scan_smem = (size_t)(plan.chunk / (1 << sa.page_shift) + 1) * 4;
  e = configure_kernel((const void*)scan_kernel<D, R>, (int)scan_smem, false);
  if (e != cudaSuccess) return e;
  e = launch_k(scan_kernel<D, R>, dim3(plan.n_chunks, pairs), scan_smem, true, s, sa);
  if (e != cudaSuccess) return e;
  const size_t sel_smem = (size_t)kSelectCap * 8;
  e = configure_kernel((const void*)select_kernel<D, R>, (int)sel_smem, false);
  if (e != cudaSuccess) return e;
  return launch_k(select_kernel<D, R>, dim3(pairs), sel_smem, true, s, sel);
}

}  // namespace score_detail

ScorePlan plan_score(int pairs, int max_seq_len, int page_size) {
  using namespace score_detail;
  ScorePlan p;
  // positions per scan CTA: a power of two in [2048, 8192] and a multiple of the page size,
  // smaller while the grid would not cover every SM several times over
  int chunk = 8192;
  while (chunk > 2048 && (long long)pairs * ((max_seq_len + chunk - 1) / chunk) < 6LL * num_sms())
    chunk >>= 1;
  while (chunk % page_size) chunk <<= 1;
  while ((long long)((max_seq_len + chunk - 1) / chunk) * kWarps > kMaxRegions) chunk <<= 1;
  p.chunk = chunk;
  p.n_chunks = (max_seq_len + chunk - 1) / chunk;
  if (p.n_chunks < 1) p.n_chunks = 1;
  const size_t prep = (size_t)pairs * kPrepBytes;
  const size_t counts = ((size_t)pairs * p.n_chunks * kWarps * 4 + 255) / 256 * 256;
  const size_t entries = (size_t)pairs * p.n_chunks * chunk;
  p.ws_bytes = prep + counts + entries * 8;
  return p;
}

cudaError_t launch_score_topk(const uint16_t* q, const float* basis, const uint8_t* score_cache,
                              const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                              int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                              int page_size, int budget, int32_t* idx, int32_t* count, void* ws,
                              int* attend_tickets, const StoreNew* store, bool pdl,
                              cudaStream_t s) {
  using namespace score_detail;
  const int pairs = batch * h_kv;
  if (pairs == 0) return cudaSuccess;
  const ScorePlan plan = plan_score(pairs, max_pages * page_size, page_size);
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const Prep prep{w};
  const size_t counts = ((size_t)pairs * plan.n_chunks * kWarps * 4 + 255) / 256 * 256;
  const size_t entries = (size_t)pairs * plan.n_chunks * plan.chunk;
  Cands cands;
  cands.cnt = reinterpret_cast<uint32_t*>(w + (size_t)pairs * kPrepBytes);
  cands.key = reinterpret_cast<uint32_t*>(w + (size_t)pairs * kPrepBytes + counts);
  cands.pos = reinterpret_cast<int32_t*>(w + (size_t)pairs * kPrepBytes + counts + entries * 4);
  cands.attend_tickets = attend_tickets;

  PrepArgs pa = {};
  pa.q = q; pa.basis = basis; pa.score_cache = score_cache;
  pa.block_table = block_table; pa.max_pages = max_pages; pa.seq_lens = seq_lens;
  pa.h_q = h_q; pa.h_kv = h_kv; pa.num_pages = num_pages; pa.page_shift = shift;
  pa.budget = budget; pa.prep = prep;
  if (store) pa.store = *store;
  ScanArgs sa = {};
  sa.score_cache = score_cache; sa.block_table = block_table; sa.max_pages = max_pages;
  sa.seq_lens = seq_lens; sa.h_kv = h_kv; sa.num_pages = num_pages; sa.page_shift = shift;
  sa.chunk = plan.chunk; sa.n_chunks = plan.n_chunks; sa.budget = budget; sa.prep = prep;
  sa.cands = cands;
  const SelectArgs sel = {sa, idx, count};
  if (d == 128 && r == 32)
    return score_detail::launch_t<128, 32>(plan, pairs, pa, sa, sel, store != nullptr, pdl, s);
  if (d == 128 && r == 64)
    return score_detail::launch_t<128, 64>(plan, pairs, pa, sa, sel, store != nullptr, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
