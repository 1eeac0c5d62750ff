// Score + top-B (JSSA summary, eq. (1) and section 3.1 steps 1-2; JSSA README, section 4:
// jssa_budget tokens per decode step and KV head). Three kernels, chained on one stream with
// programmatic dependent launch:
//
// prep   one CTA per (sequence, KV head). p = M_h qbar (qbar = mean of the G query heads of KV
//        head h) in fp32, written as a sum of two f16 "digit" vectors with power-of-two weights,
//        p ~ 2^-e0 D0 + 2^-e1 D1 (D1 rounds what D0 left; about 22 significant bits of every
//        component relative to the largest one). BF16 codes use four bf16 digits instead. Then a
//        candidate threshold: a stratified sample of 2048 positions (512 strata, a run of 4
//        consecutive positions in each) is scored exactly as the scan scores, and the k-th
//        largest sampled key, k = ceil(E + 4 sqrt(E) + 8) with E = B * 2048 / L, is found by
//        histograms spaced evenly in score over the sample's range, refined until the bin that
//        holds it has at most 256 keys, which are ranked against each other. The threshold only
//        decides which keys travel to the select kernel; the selection itself is exact. At decode
//        the same kernel first stores the new token: its K and V rows and its scoring code
//        e4m3(M_h k) (float64 sum, one rounding).
// scan   CTAs over (chunk of positions, sequence x KV head): a stream of the FP8 scoring rows,
//        page-table indexed. Each of the 8 warps walks a contiguous run of 16-token tiles through
//        its own ring of shared-memory stages filled by 16-byte cp.async copies (3 stages at
//        32-byte rows, 4 at 64-byte rows, 2 at 128-byte rows), all but one stage in flight ahead
//        of the tile being scored. The codes are widened exactly to f16 (cvt e4m3x2 -> f16x2) and
//        multiplied by the two digit vectors on the tensor cores (mma.sync m16n8k16, fp32
//        accumulation); every lane ends up with one complete score. Keys at or above the
//        threshold are appended with their positions, in position order, to the warp's region.
// select one CTA per (sequence, KV head): the exact budget-th largest key among the candidates
//        and the ordered emission of the index set (keys above it, then equal keys in position
//        order up to the budget: ties go to the lower position), ascending. Three tiers: the
//        candidates of up to 128 regions held in registers, up to 6144 candidates flattened into
//        registers, or candidates staged in shared memory (or read in place) with a general
//        histogram / radix selection. If the candidates are fewer than the budget (the sampled
//        threshold was too high -- not expected in practice), the CTA first rescans the sequence
//        with no threshold, so the result is exact in every case.
// seq_len <= budget selects every position without scoring.
#include <cuda_fp16.h>

#include "common.cuh"

namespace jssa {

namespace score_detail {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnrollBytes = 32;   // bytes of scoring rows per lane per load batch
constexpr int kBins = 2048;
constexpr int kSample = 2048;      // sampled positions per (sequence, KV head), up to 64-byte rows
constexpr int kExactMax = 16384;   // up to this context every token is a candidate
constexpr int kSelectCap = 16384;  // candidates the select kernel stages in shared memory
constexpr int kRegionsPerChunk = kWarps;  // candidate regions (one per scan warp) per chunk
constexpr int kMaxRegions = 4096;  // candidate regions per (sequence, KV head)
constexpr int kPrepBytes = 1024;   // per (sequence, KV head): digits, scales, threshold, mode
constexpr int kPrepScale = 512, kPrepThr = 544, kPrepMode = 548, kPrepKmax = 552;
constexpr int kModeScan = 0, kModeAll = 1;

// Scoring-cache code format: E4M3, one byte per projected dimension (the method's cache), or
// BF16, two bytes (the ablation the FP8 choice is compared with; JSSA README, section 4 notes,
// and JSSA summary, section 3.4). A row of R codes is split over the 4 lanes of a quad.
template <int R_, bool BF16_>
struct Codes {
  static constexpr int R = R_;
  static constexpr bool kBF16 = BF16_;
  static constexpr int kBytes = BF16_ ? 2 * R_ : R_;  // per token
  static constexpr int kLaneBytes = kBytes / 4;        // one lane's share of a row
  static constexpr int kRegs = kLaneBytes / 4;         // 32-bit registers per row per lane
  static constexpr int kDigits = BF16_ ? 4 : 2;        // digit vectors of p
};

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Block-wide (NT threads): the bin of s_hist[0:nb) that holds the want-th largest element
// counted from the top bin down, the number of elements in strictly higher bins and the bin's
// own count, in s_info[0..2] (s_info[3] = 1 when found). Every thread sums nb / NT adjacent
// bins, then an exclusive scan over the threads (top bins first) finds the one thread whose
// range holds it.
template <int NT>
__device__ void find_bin(const uint32_t* s_hist, int nb, uint32_t want, uint32_t* s_wsum,
                         int* s_info) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bpt = nb > NT ? nb / NT : 1;
  const int hi = nb - tid * bpt;
  const int lo = max(0, hi - bpt);
  uint32_t c = 0;
  for (int j = lo; j < hi; ++j) c += s_hist[j];
  const uint32_t incl_w = warp_incl_scan(c, lane);
  if (lane == 31) s_wsum[warp] = incl_w;
  if (tid == 0) s_info[3] = 0;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp; ++w) before += s_wsum[w];
  const uint32_t excl = before + incl_w - c;
  if (hi > lo && excl < want && excl + c >= want) {
    uint32_t run = excl;
    for (int j = hi - 1; j >= lo; --j) {
      const uint32_t cj = s_hist[j];
      if (run + cj >= want) {
        s_info[0] = j;
        s_info[1] = (int)run;
        s_info[2] = (int)cj;
        s_info[3] = 1;
        break;
      }
      run += cj;
    }
  }
  __syncthreads();
}

// Block-wide (NT threads) min and max of per-thread values (s_red: 2 * NT / 32 words).
template <int NT>
__device__ __forceinline__ void block_min_max(uint32_t& mn, uint32_t& mx, uint32_t* s_red) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) {
    s_red[warp] = mn;
    s_red[NW + warp] = mx;
  }
  __syncthreads();
  mn = s_red[0];
  mx = s_red[NW];
  for (int w = 1; w < NW; ++w) {
    mn = min(mn, s_red[w]);
    mx = max(mx, s_red[NW + w]);
  }
  __syncthreads();
}

// Block-wide (NT threads) exclusive prefix of a per-thread 64-bit value; returns the prefix and
// the total (s_red: NT / 32 words of 64 bits).
template <int NT>
__device__ __forceinline__ uint64_t block_excl_scan64(uint64_t v, uint64_t& total, uint64_t* s_red) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_red[warp] = x;
  __syncthreads();
  uint64_t before = 0;
  total = 0;
  for (int w = 0; w < NW; ++w) {
    const uint64_t t = s_red[w];
    if (w < warp) before += t;
    total += t;
  }
  __syncthreads();
  return before + x - v;
}

// Radix select over n keys read through key_at(i), all in [kmin, kmax]: the digits are taken
// from v = key - kmin, starting at the highest bit of kmax - kmin, at most 11 bits a pass, so
// the first histogram already spreads the keys over the range they occupy. On return the want
// largest keys are the keys > thr plus `take` of the keys == thr (exact result), unless
// max_passes ran out first: then take = 0 and the keys > thr are a superset of them (the lowest
// key of the bin that holds the want-th largest is thr + 1). Block-wide (NT threads); s_hist:
// 2048 words, s_wsum: NT / 32 words.
template <int NT, typename KeyAt>
__device__ void radix_select(KeyAt key_at, int n, uint32_t want, uint32_t kmin, uint32_t kmax,
                             int max_passes, uint32_t* s_hist, uint32_t* s_wsum, int* s_info,
                             int64_t& thr, uint32_t& take) {
  const int tid = threadIdx.x;
  int bits = 32 - __clz(kmax - kmin);  // 0 when every key is equal
  uint32_t prefix = 0;                 // the digits decided so far (bits above `bits`)
  if (bits == 0 || want == 0) {
    thr = (int64_t)kmin;
    take = want;
    if (want == 0) thr = (int64_t)kmax;
    return;
  }
#pragma unroll 1
  for (int pass = 0;; ++pass) {
    const int dbits = min(11, bits);
    const int shift = bits - dbits;
    const int nb = 1 << dbits;
    for (int i = tid; i < nb; i += NT) s_hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += NT) {
      const uint32_t v = key_at(i) - kmin;
      if ((uint32_t)((uint64_t)v >> bits) == prefix)
        atomicAdd(&s_hist[(v >> shift) & (uint32_t)(nb - 1)], 1u);
    }
    __syncthreads();
    find_bin<NT>(s_hist, nb, want, s_wsum, s_info);
    if (!s_info[3]) {  // fewer keys than want: inconsistent input, select every key
      if (tid == 0) raise_flag(8u);
      thr = (int64_t)kmin - 1;
      take = 0;
      return;
    }
    want -= (uint32_t)s_info[1];
    prefix = (prefix << dbits) | (uint32_t)s_info[0];
    bits = shift;
    const uint32_t in_bin = (uint32_t)s_info[2];
    __syncthreads();  // s_info and s_hist are reused by the next pass
    if (want == in_bin || (bits > 0 && pass + 1 == max_passes)) {
      // the whole bin (or, out of passes, a superset): every key >= its lowest key
      thr = (int64_t)kmin + ((int64_t)prefix << bits) - 1;
      take = 0;
      return;
    }
    if (bits == 0) {
      thr = (int64_t)kmin + prefix;
      take = want;
      return;
    }
  }
}

// Exact threshold for the want largest of n keys in [kmin, kmax] (same contract as
// radix_select): one 11-bit histogram pass over the key range finds the bin that holds the
// want-th largest key; a bin taken whole ends it, and a bin of at most 256 keys is resolved by
// ranking its keys against each other in shared memory; larger bins fall back to radix_select.
template <int NT, typename KeyAt>
__device__ void select_threshold(KeyAt key_at, int n, uint32_t want, uint32_t kmin, uint32_t kmax,
                                 uint32_t* s_hist, uint32_t* s_wsum, int* s_info, int64_t& thr,
                                 uint32_t& take) {
  const int tid = threadIdx.x;
  const int bits = 32 - __clz(kmax - kmin);
  if (bits <= 11 || want == 0) {
    radix_select<NT>(key_at, n, want, kmin, kmax, 3, s_hist, s_wsum, s_info, thr, take);
    return;
  }
  const int shift = bits - 11;
  for (int i = tid; i < kBins; i += NT) s_hist[i] = 0u;
  __syncthreads();
  for (int i = tid; i < n; i += NT) atomicAdd(&s_hist[(key_at(i) - kmin) >> shift], 1u);
  __syncthreads();
  find_bin<NT>(s_hist, kBins, want, s_wsum, s_info);
  if (!s_info[3]) {  // fewer keys than want: inconsistent input, select every key
    if (tid == 0) raise_flag(8u);
    thr = (int64_t)kmin - 1;
    take = 0;
    return;
  }
  const uint32_t bin = (uint32_t)s_info[0], m = (uint32_t)s_info[2];
  const uint32_t w2 = want - (uint32_t)s_info[1];
  __syncthreads();  // s_info and s_hist are reused below
  if (w2 == m) {
    thr = (int64_t)kmin + ((int64_t)bin << shift) - 1;
    take = 0;
    return;
  }
  if (m > 256) {
    radix_select<NT>(key_at, n, want, kmin, kmax, 3, s_hist, s_wsum, s_info, thr, take);
    return;
  }
  if (tid == 0) s_info[3] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += NT) {
    const uint32_t key = key_at(i);
    if (((key - kmin) >> shift) == bin) s_hist[atomicAdd(&s_info[3], 1)] = key;
  }
  __syncthreads();
  if (tid < (int)m) {
    const uint32_t x = s_hist[tid];
    uint32_t gt = 0, eq = 0;
    for (uint32_t j = 0; j < m; ++j) {
      const uint32_t y = s_hist[j];
      gt += y > x;
      eq += y == x;
    }
    if (gt < w2 && w2 <= gt + eq) {  // x is the w2-th largest of the bin (equal keys agree)
      s_info[0] = (int)x;
      s_info[1] = (int)(w2 - gt);
    }
  }
  __syncthreads();
  thr = (int64_t)(uint32_t)s_info[0];
  take = (uint32_t)s_info[1];
  __syncthreads();
}

// Exact threshold (contract of radix_select) from a histogram of the n keys built beforehand
// with bin(key) = min(NB - 1, (key - base) >> shift), every key >= base: the bin of the want-th
// largest key, taken whole or resolved by ranking its keys (at most 256) against each other.
// Returns false, leaving thr / take unset, when that bin is the top one (it also holds every key
// above the range) or holds more keys: the caller then runs a general selection.
template <int NT, int NB, typename KeyAt>
__device__ bool threshold_from_hist(KeyAt key_at, int n, uint32_t want, uint32_t base, int shift,
                                    uint32_t* s_hist, uint32_t* s_wsum, int* s_info, int64_t& thr,
                                    uint32_t& take) {
  const int tid = threadIdx.x;
  find_bin<NT>(s_hist, NB, want, s_wsum, s_info);
  const bool found = s_info[3] != 0;
  const uint32_t bin = (uint32_t)s_info[0], m = (uint32_t)s_info[2];
  const uint32_t w2 = want - (uint32_t)s_info[1];
  __syncthreads();  // s_info and s_hist are reused below
  if (!found || bin == NB - 1 || (w2 != m && m > 256)) return false;
  if (w2 == m) {
    thr = (int64_t)base + ((int64_t)bin << shift) - 1;
    take = 0;
    return true;
  }
  if (tid == 0) s_info[3] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += NT) {
    const uint32_t key = key_at(i);
    if (((key - base) >> shift) == bin) s_hist[atomicAdd(&s_info[3], 1)] = key;
  }
  __syncthreads();
  if (tid < (int)m) {
    const uint32_t x = s_hist[tid];
    uint32_t gt = 0, eq = 0;
    for (uint32_t j = 0; j < m; ++j) {
      const uint32_t y = s_hist[j];
      gt += y > x;
      eq += y == x;
    }
    if (gt < w2 && w2 <= gt + eq) {  // x is the w2-th largest of the bin (equal keys agree)
      s_info[0] = (int)x;
      s_info[1] = (int)(w2 - gt);
    }
  }
  __syncthreads();
  thr = (int64_t)(uint32_t)s_info[0];
  take = (uint32_t)s_info[1];
  __syncthreads();
  return true;
}

// The score a key was made from (score_key inverted); keys below the key of the lowest finite
// score (unusable samples) give -inf.
__device__ __forceinline__ float key_value(uint32_t key) {
  if (key < 0x00800000u) return -INFINITY;
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// The k-th largest of the sampled keys, NK of them in each thread's registers; [kmin, kmax] is
// the range of the keys of finite scores. Each pass histograms the keys still in play (all at
// first, then those of the bin picked last) into NB bins spaced evenly in score over their range
// (score keys are not linear in the score: one bin range in key space spans every binade of the
// small scores near zero), finds the bin that holds the wanted key, and stops when that bin holds
// at most 256 keys, which are then ranked against each other. Keys below kmin fall into the
// lowest bin. s_hist (NB words) is zero on entry; s_list holds 256 keys; *s_nlist is zero on
// entry. Every thread returns the same value. Block-wide (NT threads).
template <int NT, int NB, int NK>
__device__ uint32_t sample_threshold(const uint32_t (&key)[NK], uint32_t k, uint32_t kmin,
                                     uint32_t kmax, uint32_t* s_hist, uint32_t* s_list,
                                     int* s_nlist, uint32_t* s_wsum, int* s_info) {
  static_assert(NB <= NT * 8 && (NB & (NB - 1)) == 0, "histogram size");
  constexpr int kLog = NB == 256 ? 8 : NB == 512 ? 9 : NB == 1024 ? 10 : 11;
  const int tid = threadIdx.x;
  uint32_t live = (1u << NK) - 1u;  // bit j: key[j] is in the bin being refined
  uint32_t lo = kmin, hi = kmax;    // key range of the live keys (of finite scores)
  uint32_t want = k;                // rank of the wanted key among the live keys
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    if (hi <= lo) return hi;  // one key value left (or no finite score at all)
    const float vlo = key_value(lo), vhi = key_value(hi);
    const float scale = (float)NB / (vhi - vlo);
    // bins evenly spaced in score; in key space when the score range is not representable
    const bool linear = isfinite(vhi - vlo) && isfinite(scale) && scale > 0.f;
    const int kshift = max(0, 32 - kLog - __clz(hi - lo));  // key space: at most NB bins
    int kb[NK];
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      if (linear)
        kb[j] = min(NB - 1, (int)fmaxf(0.f, (key_value(key[j]) - vlo) * scale));
      else
        kb[j] = key[j] < lo ? 0 : min(NB - 1, (int)((key[j] - lo) >> kshift));
    }
    if (pass > 0) {
      for (int i = tid; i < NB; i += NT) s_hist[i] = 0u;
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < NK; ++j)
      if (live >> j & 1u) atomicAdd(&s_hist[kb[j]], 1u);
    __syncthreads();
    find_bin<NT>(s_hist, NB, want, s_wsum, s_info);
    if (!s_info[3]) {  // fewer keys than wanted: inconsistent input, every key qualifies
      if (tid == 0) raise_flag(8u);
      return 0u;
    }
    const int bin = s_info[0];
    want -= (uint32_t)s_info[1];
    const uint32_t m = (uint32_t)s_info[2];
#pragma unroll
    for (int j = 0; j < NK; ++j)
      if (kb[j] != bin) live &= ~(1u << j);
    if (m <= 256) {
      // rank the bin's keys: the want-th largest of them (equal keys agree)
#pragma unroll
      for (int j = 0; j < NK; ++j)
        if (live >> j & 1u) s_list[atomicAdd(s_nlist, 1)] = key[j];
      __syncthreads();
      if (tid < (int)m) {
        const uint32_t x = s_list[tid];
        uint32_t gt = 0, eq = 0;
        for (uint32_t i = 0; i < m; ++i) {
          const uint32_t y = s_list[i];
          gt += y > x;
          eq += y == x;
        }
        if (gt < want && want <= gt + eq) s_info[0] = (int)x;
      }
      __syncthreads();
      return (uint32_t)s_info[0];
    }
    // the next pass spreads the picked bin's keys over the whole histogram
    uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
    for (int j = 0; j < NK; ++j)
      if (live >> j & 1u) {
        mn = min(mn, key[j]);
        mx = max(mx, key[j]);
      }
    block_min_max<NT>(mn, mx, s_wsum);  // (its barriers also retire s_hist and s_info)
    lo = mn;
    hi = mx;
  }
  return lo;  // still more than 256 keys in play: the lowest of them (a superset threshold)
}

struct Prep {
  uint8_t* rec;  // [pairs][kPrepBytes]: digits [8][R] at 0, scales at kPrepScale, threshold
                 // key at kPrepThr, mode at kPrepMode
};
struct Cands {
  uint32_t* key;       // [pairs][n_chunks][kRegionsPerChunk][chunk / kRegionsPerChunk]
  int32_t* pos;        // same layout
  uint32_t* cnt;       // [pairs][n_chunks][kRegionsPerChunk]
  int* attend_tickets; // [pairs][tickets_per_pair] split-K tickets of the attention that follows,
                       // or null
  int tickets_per_pair;
};

// The select of a pair clears the split-K tickets the attention that follows uses for it.
__device__ __forceinline__ void clear_attend_tickets(const Cands& c, int pair) {
  if (!c.attend_tickets) return;
  for (int i = threadIdx.x; i < c.tickets_per_pair; i += blockDim.x)
    c.attend_tickets[(int64_t)pair * c.tickets_per_pair + i] = 0;
}

__device__ __forceinline__ uint32_t mix32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}

// Fragment registers of the digit matrix (B operand of mma m16n8k16: f16 digits for E4M3 codes,
// bf16 digits for BF16 codes). Column n holds digit n & 1 (the two digits repeated four times;
// BF16 codes use a second set for digits 2 and 3), so lane (g, t) finds the complete digit sums
// of its rows in accumulator columns 2t and 2t + 1. K-slots are permuted so that each lane's MMA
// operands come from its own code bytes: in k-block kb (16 slots), slots 2t, 2t+1, 2t+8, 2t+9
// <-> dimensions t*R/4 + 4kb + 0..3 of the row; the same permutation on both operands leaves the
// dot products unchanged.
template <class C>
struct DigitFrags {
  static constexpr int R = C::R, KB = R / 16;
  uint32_t b0[KB], b1[KB];                              // digits 0 and 1
  uint32_t b2[C::kBF16 ? KB : 1], b3[C::kBF16 ? KB : 1];  // digits 2 and 3 (BF16 codes)
  float sc[C::kDigits];
  // dig: 16-bit digits [kDigits][R]; scale: the power-of-two weight of each digit
  __device__ __forceinline__ void load(const uint16_t* dig, const float* scale, int lane) {
    constexpr int LD = R / 4;  // dimensions per lane
    const int g = lane >> 2, t = lane & 3;
    const uint16_t* d = dig + (g & 1) * R;
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
      const int o = t * LD + 4 * kb;
      b0[kb] = (uint32_t)d[o] | ((uint32_t)d[o + 1] << 16);
      b1[kb] = (uint32_t)d[o + 2] | ((uint32_t)d[o + 3] << 16);
      if (C::kBF16) {
        const uint16_t* d2 = d + 2 * R;
        b2[kb] = (uint32_t)d2[o] | ((uint32_t)d2[o + 1] << 16);
        b3[kb] = (uint32_t)d2[o + 2] | ((uint32_t)d2[o + 3] << 16);
      }
    }
#pragma unroll
    for (int c = 0; c < C::kDigits; ++c) sc[c] = scale[c];
  }
};

// A lane's LB code bytes of one row: from shared memory through a generic pointer, from shared
// memory by shared-window address, and from global memory (streamed, no L1 allocation).
template <int LB>
__device__ __forceinline__ void load_srow(uint32_t* dst, const uint8_t* src) {
  if (LB == 4) {
    dst[0] = *reinterpret_cast<const uint32_t*>(src);
  } else if (LB == 8) {
    const uint2 v = *reinterpret_cast<const uint2*>(src);
    dst[0] = v.x;
    dst[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < LB / 16; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
      dst[4 * i] = v.x;
      dst[4 * i + 1] = v.y;
      dst[4 * i + 2] = v.z;
      dst[4 * i + 3] = v.w;
    }
  }
}

template <int LB>
__device__ __forceinline__ void lds_row(uint32_t* dst, uint32_t saddr) {
  if (LB == 4) {
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(dst[0]) : "r"(saddr) : "memory");
  } else if (LB == 8) {
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                 : "=r"(dst[0]), "=r"(dst[1])
                 : "r"(saddr)
                 : "memory");
  } else {
#pragma unroll
    for (int i = 0; i < LB / 16; ++i)
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(dst[4 * i]), "=r"(dst[4 * i + 1]), "=r"(dst[4 * i + 2]),
                     "=r"(dst[4 * i + 3])
                   : "r"(saddr + 16 * i)
                   : "memory");
  }
}

template <int LB>
__device__ __forceinline__ void load_row(uint32_t* dst, const uint8_t* src) {
  if (LB == 4) {
    dst[0] = __ldcs(reinterpret_cast<const unsigned int*>(src));
  } else if (LB == 8) {
    const uint2 v = ld_stream_v2(src);
    dst[0] = v.x;
    dst[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < LB / 16; ++i) {
      const uint4 v = ld_stream_v4(src + 16 * i);
      dst[4 * i] = v.x;
      dst[4 * i + 1] = v.y;
      dst[4 * i + 2] = v.z;
      dst[4 * i + 3] = v.w;
    }
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

template <class C>
struct ScanBuf {
  // tiles per batch (even)
  static constexpr int kUnroll = kUnrollBytes / C::kLaneBytes > 2 ? kUnrollBytes / C::kLaneBytes : 2;
  uint32_t ra[kUnroll][C::kRegs], rb[kUnroll][C::kRegs];
  uint32_t ok;  // bit u: tile u is inside the run and the chunk and its page is usable
};

// Rows of tiles [t0, t0 + kUnroll) (rows g and g+8 of each tile for lane (g, t)). The loads are
// unconditional: a tile past t_end or the chunk's valid tokens, or on an unusable page, reads
// page 0 instead (always allocated) and its tokens are never candidates (see scan_emit).
// BIG: pages of at least 16 tokens, so a tile lies inside one page.
template <class C, bool BIG>
__device__ __forceinline__ void scan_load(ScanBuf<C>& buf, const ChunkGeom& cg,
                                          const int32_t* s_page, int t0, int t_end, int lane) {
  constexpr int LB = C::kLaneBytes, RB = C::kBytes;
  const int g = lane >> 2, t = lane & 3;
  const int pmask = (1 << cg.page_shift) - 1;
  if (BIG) {
    const int lane_off = g * RB + t * LB;
    buf.ok = 0u;
#pragma unroll
    for (int u = 0; u < ScanBuf<C>::kUnroll; ++u) {
      const int tok0 = (t0 + u) * 16;
      const int pg = t0 + u < t_end && tok0 < cg.n_local ? s_page[tok0 >> cg.page_shift] : -1;
      buf.ok |= (uint32_t)(pg >= 0) << u;
      const uint8_t* row = cg.head_base + (size_t)(uint32_t)max(pg, 0) * cg.page_bytes +
                           ((tok0 & pmask) * RB + lane_off);
      load_row<LB>(buf.ra[u], row);
      load_row<LB>(buf.rb[u], row + 8 * RB);
    }
  } else {
    buf.ok = ~0u;  // token validity is checked per token at emission
#pragma unroll
    for (int u = 0; u < ScanBuf<C>::kUnroll; ++u) {
      const bool live = t0 + u < t_end;
      const int ta = (t0 + u) * 16 + g, tb = ta + 8;
      const int pa = live && ta < cg.n_local ? s_page[ta >> cg.page_shift] : 0;
      const int pb = live && tb < cg.n_local ? s_page[tb >> cg.page_shift] : 0;
      load_row<LB>(buf.ra[u], cg.head_base + (size_t)(uint32_t)max(pa, 0) * cg.page_bytes +
                                  ((ta & pmask) * RB + t * LB));
      load_row<LB>(buf.rb[u], cg.head_base + (size_t)(uint32_t)max(pb, 0) * cg.page_bytes +
                                  ((tb & pmask) * RB + t * LB));
    }
  }
}

// Scores of two 16-token tiles, one token per lane: lane (g, t) returns token
// 16 * (t >> 1) + 8 * (t & 1) + g of the pair. ra / rb hold the lane's code bytes of rows g and
// g + 8 (a quarter of a row each). E4M3 codes are widened to f16 (exact) and multiplied by the
// f16 digits, BF16 codes are multiplied as they are by the bf16 digits, on the tensor cores with
// fp32 accumulation: s = sum_c 2^-e_c C_c (c over the digits).
template <class C>
__device__ __forceinline__ float pair_scores(const uint32_t* ra0, const uint32_t* rb0,
                                             const uint32_t* ra1, const uint32_t* rb1,
                                             const DigitFrags<C>& df, int t) {
  constexpr int KB = C::R / 16;
  float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
  float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) {
    if (C::kBF16) {
      mma_bf16(c0, ra0[2 * kb], rb0[2 * kb], ra0[2 * kb + 1], rb0[2 * kb + 1], df.b0[kb], df.b1[kb]);
      mma_bf16(c1, ra1[2 * kb], rb1[2 * kb], ra1[2 * kb + 1], rb1[2 * kb + 1], df.b0[kb], df.b1[kb]);
      mma_bf16(e0, ra0[2 * kb], rb0[2 * kb], ra0[2 * kb + 1], rb0[2 * kb + 1], df.b2[kb], df.b3[kb]);
      mma_bf16(e1, ra1[2 * kb], rb1[2 * kb], ra1[2 * kb + 1], rb1[2 * kb + 1], df.b2[kb], df.b3[kb]);
    } else {
      mma_f16(c0, e4m3x2_to_f16x2((uint16_t)ra0[kb]), e4m3x2_to_f16x2((uint16_t)rb0[kb]),
              e4m3x2_to_f16x2((uint16_t)(ra0[kb] >> 16)), e4m3x2_to_f16x2((uint16_t)(rb0[kb] >> 16)),
              df.b0[kb], df.b1[kb]);
      mma_f16(c1, e4m3x2_to_f16x2((uint16_t)ra1[kb]), e4m3x2_to_f16x2((uint16_t)rb1[kb]),
              e4m3x2_to_f16x2((uint16_t)(ra1[kb] >> 16)), e4m3x2_to_f16x2((uint16_t)(rb1[kb] >> 16)),
              df.b0[kb], df.b1[kb]);
    }
  }
  const bool hi_row = t & 1, tile1 = t & 2;
  const float x0 = hi_row ? c0[2] : c0[0], y0 = hi_row ? c0[3] : c0[1];
  const float x1 = hi_row ? c1[2] : c1[0], y1 = hi_row ? c1[3] : c1[1];
  float f = (tile1 ? x1 : x0) * df.sc[0] + (tile1 ? y1 : y0) * df.sc[1];
  if (C::kBF16) {
    const float u0 = hi_row ? e0[2] : e0[0], v0 = hi_row ? e0[3] : e0[1];
    const float u1 = hi_row ? e1[2] : e1[0], v1 = hi_row ? e1[3] : e1[1];
    f += (tile1 ? u1 : u0) * df.sc[C::kDigits - 2] + (tile1 ? v1 : v0) * df.sc[C::kDigits - 1];
  }
  return f;
}

// The smallest float whose key is >= thr (keys of non-NaN floats are >= thr exactly when the
// float is >= it); -inf when every key qualifies.
__device__ __forceinline__ float key_floor(uint32_t thr) {
  if (thr <= 0x007FFFFFu) return -INFINITY;  // at or below the key of -inf
  const uint32_t u = (thr & 0x80000000u) ? (thr & 0x7FFFFFFFu) : ~thr;
  return __uint_as_float(u);
}

// Keys >= thr of the tiles [t0, t0 + kUnroll) appended in position order to this warp's region.
template <class C, bool BIG>
__device__ __forceinline__ void scan_emit(const ScanBuf<C>& buf, const DigitFrags<C>& df,
                                          const ChunkGeom& cg, const int32_t* s_page, int t0,
                                          int t_end, float thr_f, uint32_t* rkey, int32_t* rpos,
                                          uint32_t& run, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int tok_in_pair = 16 * (t >> 1) + 8 * (t & 1) + g;
  // lanes holding earlier tokens of the pair: every lane of a lower t, and lower g for this t
  const unsigned quad_t = 0x11111111u << t;
  const unsigned earlier_t = 0x11111111u * ((1u << t) - 1u);
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int u = 0; u < ScanBuf<C>::kUnroll; u += 2) {
    const float f = pair_scores<C>(buf.ra[u], buf.rb[u], buf.ra[u + 1], buf.rb[u + 1], df, t);
    const int tok = (t0 + u) * 16 + tok_in_pair;
    bool c = f >= thr_f && tok < cg.n_local;
    if (BIG) {
      c = c && ((buf.ok >> (u + (t >> 1))) & 1u);
    } else {
      c = c && t0 + u < t_end && (tok_in_pair < 16 || t0 + u + 1 < t_end) &&
          s_page[tok >> cg.page_shift] >= 0;
    }
    const unsigned m = __ballot_sync(0xffffffffu, c);
    if (m) {
      if (c) {
        const uint32_t at = run + __popc(m & earlier_t) + __popc(m & quad_t & lt);
        rkey[at] = score_key(f);
        rpos[at] = cg.start + tok;
      }
      run += __popc(m);
    }
  }
}

// One warp's contiguous run of tiles [t_begin, t_end), register double-buffered.
template <class C, bool BIG>
__device__ __forceinline__ uint32_t scan_warp(const ChunkGeom& cg, const int32_t* s_page,
                                              const DigitFrags<C>& df, float thr_f, int t_begin,
                                              int t_end, uint32_t* rkey, int32_t* rpos, int lane) {
  constexpr int kU = ScanBuf<C>::kUnroll;
  uint32_t run = 0;
  ScanBuf<C> a, b;
  int t0 = t_begin;
  if (t0 < t_end) scan_load<C, BIG>(a, cg, s_page, t0, t_end, lane);
  while (t0 < t_end) {
    if (t0 + kU < t_end) scan_load<C, BIG>(b, cg, s_page, t0 + kU, t_end, lane);
    scan_emit<C, BIG>(a, df, cg, s_page, t0, t_end, thr_f, rkey, rpos, run, lane);
    t0 += kU;
    if (t0 >= t_end) break;
    if (t0 + kU < t_end) scan_load<C, BIG>(a, cg, s_page, t0 + kU, t_end, lane);
    scan_emit<C, BIG>(b, df, cg, s_page, t0, t_end, thr_f, rkey, rpos, run, lane);
    t0 += kU;
  }
  return run;
}

// The scan kernel's warps stream their tiles through a ring of scan_stages<C>() shared-memory
// stages (kUnroll tiles each) filled by asynchronous 16-byte copies, all but one stage ahead of
// the one being scored: deeper than a register double buffer without holding the rows in
// registers. 16- and 32-byte rows: three stages and four CTAs per SM; 64-byte rows: four stages
// and three; 128-byte rows (the latent scoring of multi-head latent attention): two stages and
// three.
template <class C>
constexpr int scan_stage_bytes() { return ScanBuf<C>::kUnroll * 16 * C::kBytes; }
template <class C>
constexpr int scan_stages() { return C::kBytes <= 32 ? 3 : C::kBytes == 64 ? 4 : 2; }
template <class C>
constexpr int scan_ctas_per_sm() { return C::kBytes <= 32 ? 4 : 3; }
template <class C>
constexpr int scan_ring_bytes() { return kWarps * scan_stages<C>() * scan_stage_bytes<C>(); }

// Copies of tiles [t0, t0 + kUnroll) into the stage at shared address `dst`; returns the tiles'
// ok bits (as scan_load). A tile past t_end or the chunk's valid tokens, or a row on an unusable
// page, is zero-filled (its tokens are never candidates, see scan_emit).
template <class C, bool BIG>
__device__ __forceinline__ uint32_t scan_issue(uint32_t dst, const ChunkGeom& cg,
                                               const int32_t* s_page, int t0, int t_end, int lane) {
  constexpr int kU = ScanBuf<C>::kUnroll;
  constexpr int RB = C::kBytes;
  constexpr int kTileBytes = 16 * RB;
  constexpr int kPieces = kTileBytes / 512;  // 16-byte copies per lane per tile
  static_assert(kU * kTileBytes == scan_stage_bytes<C>(), "stage size");
  const int pmask = (1 << cg.page_shift) - 1;
  uint32_t ok = BIG ? 0u : ~0u;
  if constexpr (kPieces == 0) {
    // tiles under 512 bytes (16-byte rows): a warp instruction copies 512 / kTileBytes whole
    // tiles, piece (32 i + lane) of the stage being tile piece / (kTileBytes / 16)
    constexpr int kPerTile = kTileBytes / 16;
    static_assert(kPerTile > 0 && 32 % kPerTile == 0 && (kU * kPerTile) % 32 == 0, "tile pieces");
#pragma unroll
    for (int i = 0; i < kU * kPerTile / 32; ++i) {
      const int piece = 32 * i + lane;
      const int u = piece / kPerTile, o = (piece % kPerTile) * 16;
      const int tok0 = (t0 + u) * 16;
      const bool live = t0 + u < t_end && tok0 < cg.n_local;
      const int tok = tok0 + o / RB;
      const int pg = live && (BIG || tok < cg.n_local) ? s_page[(BIG ? tok0 : tok) >> cg.page_shift] : -1;
      const uint8_t* src = cg.head_base + (size_t)(uint32_t)max(pg, 0) * cg.page_bytes +
                           (BIG ? (tok0 & pmask) * RB + o : (tok & pmask) * RB + o % RB);
      cp_async16(dst + u * kTileBytes + o, src, pg >= 0 ? 16 : 0);
    }
    if (BIG) {
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int tok0 = (t0 + u) * 16;
        const bool live = t0 + u < t_end && tok0 < cg.n_local;
        ok |= (uint32_t)(live && s_page[tok0 >> cg.page_shift] >= 0) << u;
      }
    }
    return ok;
  }
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int tok0 = (t0 + u) * 16;
    const bool live = t0 + u < t_end && tok0 < cg.n_local;
    if (BIG) {
      const int pg = live ? s_page[tok0 >> cg.page_shift] : -1;
      ok |= (uint32_t)(pg >= 0) << u;
      const uint8_t* tile = cg.head_base + (size_t)(uint32_t)max(pg, 0) * cg.page_bytes +
                            (tok0 & pmask) * RB;
#pragma unroll
      for (int p = 0; p < kPieces; ++p) {
        const int o = (p * 32 + lane) * 16;
        cp_async16(dst + u * kTileBytes + o, tile + o, pg >= 0 ? 16 : 0);
      }
    } else {
#pragma unroll
      for (int p = 0; p < kPieces; ++p) {
        const int o = (p * 32 + lane) * 16;
        const int tok = tok0 + o / RB;
        const int pg = live && tok < cg.n_local ? s_page[tok >> cg.page_shift] : -1;
        const uint8_t* src = cg.head_base + (size_t)(uint32_t)max(pg, 0) * cg.page_bytes +
                             ((tok & pmask) * RB + o % RB);
        cp_async16(dst + u * kTileBytes + o, src, pg >= 0 ? 16 : 0);
      }
    }
  }
  return ok;
}

// One warp's contiguous run of tiles [t_begin, t_end) through its ring (`ring`: this warp's
// scan_stages<C>() stages in shared memory).
template <class C, bool BIG>
__device__ __forceinline__ uint32_t scan_warp_ring(const ChunkGeom& cg, const int32_t* s_page,
                                                   const DigitFrags<C>& df, float thr_f,
                                                   int t_begin, int t_end, uint32_t* rkey,
                                                   int32_t* rpos, uint8_t* ring, int lane) {
  constexpr int kU = ScanBuf<C>::kUnroll;
  constexpr int S = scan_stages<C>();
  constexpr int kStageBytes = scan_stage_bytes<C>();
  constexpr uint32_t kMask = (1u << kU) - 1u;
  constexpr int LB = C::kLaneBytes, RB = C::kBytes;
  static_assert(S * kU <= 32, "ok bits");
  const int g = lane >> 2, t = lane & 3;
  const uint32_t ring_s = smem_u32(ring);
  const int n_batch = (t_end - t_begin + kU - 1) / kU;
  uint32_t ok_ring = 0u;  // stage s: bits [s * kU, s * kU + kU)
#pragma unroll
  for (int i = 0; i < S - 1; ++i) {
    if (i < n_batch)
      ok_ring |= scan_issue<C, BIG>(ring_s + i * kStageBytes, cg, s_page, t_begin + i * kU,
                                    t_end, lane) << (i * kU);
    cp_async_commit();
  }
  uint32_t run = 0;
  for (int i = 0; i < n_batch; ++i) {
    const int nx = i + S - 1;
    if (nx < n_batch) {
      const int sx = nx % S;
      const uint32_t okx = scan_issue<C, BIG>(ring_s + sx * kStageBytes, cg, s_page,
                                              t_begin + nx * kU, t_end, lane);
      ok_ring = (ok_ring & ~(kMask << (sx * kU))) | ((okx & kMask) << (sx * kU));
    }
    cp_async_commit();
    cp_async_wait<S - 1>();
    __syncwarp();
    const int st = i % S;
    const uint32_t stage = ring_s + st * kStageBytes;
    ScanBuf<C> buf;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      lds_row<LB>(buf.ra[u], stage + u * 16 * RB + g * RB + t * LB);
      lds_row<LB>(buf.rb[u], stage + u * 16 * RB + (g + 8) * RB + t * LB);
    }
    buf.ok = BIG ? (ok_ring >> (st * kU)) & kMask : ~0u;
    __syncwarp();  // the stage is refilled by the next iteration's copies
    scan_emit<C, BIG>(buf, df, cg, s_page, t_begin + i * kU, t_end, thr_f, rkey, rpos, run, lane);
  }
  cp_async_wait<0>();
  return run;
}

// Page list of a chunk into shared memory (bounds checked; -1 = unusable page); four loads per
// thread in flight at a time.
__device__ __forceinline__ void load_pages(int32_t* s_page, const int32_t* bt, int n_pages,
                                           int64_t num_pages) {
  for (int i0 = threadIdx.x; i0 < n_pages; i0 += 4 * blockDim.x) {
    int32_t pg[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * blockDim.x;
      pg[u] = i < n_pages ? bt[i] : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i >= n_pages) continue;
      if (pg[u] < 0 || (int64_t)pg[u] >= num_pages) {
        raise_flag(1u);
        pg[u] = -1;
      }
      s_page[i] = pg[u];
    }
  }
}

__device__ __forceinline__ int clamp_len(int L, int max_len) {
  if (L < 0 || L > max_len) {
    if (threadIdx.x == 0) raise_flag(4u);
    return L < 0 ? 0 : max_len;
  }
  return L;
}

// Scan of chunk c of pair `pair` on the warp-level MMA (page list already in s_page): warp
// q < kRegionsPerChunk takes the q-th eighth of the chunk and writes that region and its count.
// RING: the scan kernel's shared-memory tile rings (`ring`); otherwise register double buffers
// (the select kernel's rescan).
template <class C, bool RING>
__device__ void scan_chunk(const ScanArgs& a, int pair, int c, int L, uint32_t thr,
                           const DigitFrags<C>& df, const int32_t* s_page, uint8_t* ring) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp >= kRegionsPerChunk) return;
  const int h = pair % a.h_kv;
  ChunkGeom cg;
  cg.start = c * a.chunk;
  cg.n_local = max(0, min(a.chunk, L - cg.start));
  cg.page_shift = a.page_shift;
  cg.page_bytes = ((uint32_t)a.h_kv << a.page_shift) * C::kBytes;
  cg.head_base = a.score_cache + ((int64_t)h << a.page_shift) * C::kBytes;
  const int seg = a.chunk / kRegionsPerChunk;
  const int64_t reg = ((int64_t)pair * a.n_chunks + c) * kRegionsPerChunk + warp;
  const int n_tiles = (cg.n_local + 15) >> 4;
  const int tpw = seg / 16;
  const int t_begin = min(n_tiles, warp * tpw), t_end = min(n_tiles, t_begin + tpw);
  const float thr_f = key_floor(thr);
  uint32_t n;
  if (RING) {
    uint8_t* wr = ring + warp * scan_stages<C>() * scan_stage_bytes<C>();
    n = cg.page_shift >= 4
            ? scan_warp_ring<C, true>(cg, s_page, df, thr_f, t_begin, t_end,
                                      a.cands.key + reg * seg, a.cands.pos + reg * seg, wr, lane)
            : scan_warp_ring<C, false>(cg, s_page, df, thr_f, t_begin, t_end,
                                       a.cands.key + reg * seg, a.cands.pos + reg * seg, wr, lane);
  } else {
    n = cg.page_shift >= 4
            ? scan_warp<C, true>(cg, s_page, df, thr_f, t_begin, t_end, a.cands.key + reg * seg,
                                 a.cands.pos + reg * seg, lane)
            : scan_warp<C, false>(cg, s_page, df, thr_f, t_begin, t_end, a.cands.key + reg * seg,
                                  a.cands.pos + reg * seg, lane);
  }
  if (lane == 0) a.cands.cnt[reg] = n;
}

template <int D, class C>
__global__ void __launch_bounds__(kThreads, scan_ctas_per_sm<C>()) scan_kernel(ScanArgs a) {
  extern __shared__ __align__(16) uint8_t scan_dyn[];  // tile ring, then the page list
  int32_t* scan_pages = reinterpret_cast<int32_t*>(scan_dyn + scan_ring_bytes<C>());
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
  pdl_trigger();  // the select may be scheduled; it waits for this grid to complete
  const uint8_t* rec = a.prep.rec + (int64_t)pair * kPrepBytes;
  const int mode = *reinterpret_cast<const int*>(rec + kPrepMode);
  if (mode == kModeAll || n_local == 0) {
    if ((threadIdx.x & 31) == 0 && (threadIdx.x >> 5) < kRegionsPerChunk)
      a.cands.cnt[((int64_t)pair * a.n_chunks + c) * kRegionsPerChunk + (threadIdx.x >> 5)] = 0u;
    return;
  }
  DigitFrags<C> df;
  df.load(reinterpret_cast<const uint16_t*>(rec), reinterpret_cast<const float*>(rec + kPrepScale),
          threadIdx.x & 31);
  const uint32_t thr = *reinterpret_cast<const uint32_t*>(rec + kPrepThr);
  scan_chunk<C, true>(a, pair, c, L, thr, df, scan_pages, scan_dyn);
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

// The sample: n_groups strata of L / n_groups tokens, in each a run of kGroup consecutive
// positions (one 128-byte line of codes at r = 32) starting at a kGroup-aligned offset drawn
// from a 32-bit mix of (stratum, pair), scaled to the stratum by a high multiply; never the last
// position (the token a decode step stores right now). 2048 positions for rows of up to 64
// bytes, 1024 for 128-byte rows (the sampled rows are staged in shared memory).
constexpr int kGroup = 4;
template <class C>
constexpr int sample_size() { return C::kBytes > 64 ? kSample / 2 : kSample; }
__device__ __forceinline__ int sample_group_start(int grp, int pair, int L, int n_groups) {
  const int stratum = L / n_groups;  // >= 32 whenever the sample is drawn
  const uint32_t hsh = mix32((uint32_t)grp * 0x9E3779B9u ^ ((uint32_t)pair * 0x85EBCA6Bu + 1u));
  const int first = (grp * stratum + kGroup - 1) / kGroup;  // first aligned slot of the stratum
  return kGroup * (first + (int)__umulhi(hsh, (uint32_t)(stratum / kGroup - 1)));
}

// query rows loaded per pass: D / 8 threads x 8 dims a row
template <int D>
constexpr int q_groups() { return kThreads / (D / 8); }
constexpr int kSampleBins = 256;          // histogram bins of the sampled scores

// Multi-head latent attention (d 576 = 512 latent + 64 rotary dimensions): the basis projects the
// 512 latent dimensions only, [R - 64, 512], and the 64 rotary dimensions pass through as the last
// 64 code columns (JSSA README, section 4 notes: the MLA basis is [1, r, kv_lora_rank]; section
// 3.4 of the JSSA summary: 64 latent + 64 RoPE scoring dimensions).
template <int D>
constexpr bool latent_layer() { return D == 576; }
constexpr int kRopeDims = 64;
template <int D>
constexpr int proj_dims() { return latent_layer<D>() ? D - kRopeDims : D; }  // dims the basis reads
template <int D, class C>
constexpr int proj_rows() { return latent_layer<D>() ? C::R - kRopeDims : C::R; }  // basis rows

// M_h is staged in shared memory when it takes at most 64 KB; otherwise (the latent basis of
// multi-head latent attention, 64 x 512) the projection reads it from global memory.
template <int D, class C>
constexpr bool prep_m_in_smem() { return proj_rows<D, C>() * proj_dims<D>() * 4 <= 64 * 1024; }

// Dynamic shared memory of the prep kernel.
template <int D, class C>
struct PrepSmem {
  uint8_t rows[sample_size<C>() * C::kBytes];  // code rows of the sampled positions
  float m[prep_m_in_smem<D, C>() ? C::R * D : 1];  // M_h, row-major [R][D] (when it fits)
  float qpart[q_groups<D>()][D]; // partial sums of the group's query rows
  uint32_t list[256];            // keys of the bin that holds the threshold
  uint32_t hist[kSampleBins];
  uint8_t valid[sample_size<C>()];  // sampled position on a usable page
};

template <int D, class C, bool STORE>
__global__ void __launch_bounds__(kThreads, 2) prep_kernel(PrepArgs a) {
  constexpr int R = C::R, LB = C::kLaneBytes, RB = C::kBytes;
  constexpr int kDigits = C::kDigits;
  constexpr int kS = sample_size<C>(), kSampleGroups = kS / kGroup;
  constexpr int kTilesPerWarp = kS / 16 / kWarps;  // 16 (8 for 128-byte rows)
  extern __shared__ __align__(16) uint8_t prep_dyn[];
  PrepSmem<D, C>& sm = *reinterpret_cast<PrepSmem<D, C>*>(prep_dyn);
  __shared__ __align__(16) float s_qbar[D];
  __shared__ __align__(16) float s_k[D];
  __shared__ float s_p[R];
  __shared__ __align__(16) uint16_t s_dig[kDigits * R];  // f16 (E4M3 codes) or bf16 digits
  __shared__ float s_scale[kDigits];
  __shared__ uint32_t s_wsum[2 * kWarps];
  __shared__ int s_info[4];
  __shared__ int s_nlist;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int pair = blockIdx.x;
  const int b = pair / a.h_kv, h = pair % a.h_kv;
  const int G = a.h_q / a.h_kv;
  const int page_size = 1 << a.page_shift;
  const int32_t* bt = a.block_table + (int64_t)b * a.max_pages;
  constexpr int kPD = proj_dims<D>(), kPR = proj_rows<D, C>();
  const float* m_h = a.basis + (int64_t)h * kPR * kPD;

  // launched as a programmatic dependent of whatever precedes it on the stream: nothing is read
  // before that kernel has completed. The scan may be scheduled at once (it waits for this grid
  // before reading what it writes).
  pdl_wait();
  pdl_trigger();

  // ---- independent loads first: M_h into shared memory (async); L, the group's query rows and
  // the new token's K and V rows into registers ----
  constexpr bool kMSmem = prep_m_in_smem<D, C>();
  constexpr int kQGroups = q_groups<D>();
  {
    // a group of many query heads (the 128 heads of a latent layer) is summed over many rounds
    // of loads, and a basis too large for shared memory is read row by row: both are prefetched
    // into L2 in 4 KB pieces first, so that those rounds wait on L2 and not on HBM
    constexpr int kPiece = 4096;
    const int q_bytes = G > kQGroups ? G * D * 2 : 0;
    const int m_bytes = kMSmem ? 0 : kPR * kPD * 4;
    const int q_pieces = (q_bytes + kPiece - 1) / kPiece, m_pieces = (m_bytes + kPiece - 1) / kPiece;
    const uint8_t* q_src = reinterpret_cast<const uint8_t*>(a.q + ((int64_t)b * a.h_q + (int64_t)h * G) * D);
    const uint8_t* m_src = reinterpret_cast<const uint8_t*>(m_h);
    for (int i = tid; i < q_pieces + m_pieces; i += kThreads) {
      if (i < q_pieces) prefetch_l2_bulk(q_src + i * kPiece, min(kPiece, q_bytes - i * kPiece));
      else prefetch_l2_bulk(m_src + (i - q_pieces) * kPiece, min(kPiece, m_bytes - (i - q_pieces) * kPiece));
    }
  }
  if (kMSmem)
    for (int i = tid; i < R * D / 4; i += kThreads) cp_async16(smem_u32(sm.m + 4 * i), m_h + 4 * i, 16);
  cp_async_commit();
  const int L = clamp_len(a.seq_lens[b], a.max_pages << a.page_shift);
  // the G query rows of this KV head: D / 8 threads x 8 dims per row, kQGroups rows at a time
  static_assert(D % 8 == 0 && D / 8 <= kThreads, "query row split");
  const uint16_t* qh = a.q + ((int64_t)b * a.h_q + (int64_t)h * G) * D;
  const int rg = tid / (D / 8), d8 = (tid % (D / 8)) * 8;
  uint4 qv = make_uint4(0u, 0u, 0u, 0u);
  if (rg < kQGroups && rg < G) qv = *reinterpret_cast<const uint4*>(qh + (int64_t)rg * D + d8);
  const bool store = STORE && L > 0;
  constexpr int KE = (D + kThreads - 1) / kThreads;  // elements of the new K / V rows per thread
  uint16_t k_el[KE], v_el[KE];                        // elements tid, tid + kThreads, ...
#pragma unroll
  for (int u = 0; u < KE; ++u) {
    const int i = tid + u * kThreads;
    k_el[u] = v_el[u] = 0;
    if (STORE && i < D) {
      k_el[u] = a.store.k_new[((int64_t)b * a.h_kv + h) * D + i];
      if (a.store.v_new) v_el[u] = a.store.v_new[((int64_t)b * a.h_kv + h) * D + i];
    }
  }
  for (int i = tid; i < kSampleBins; i += kThreads) sm.hist[i] = 0u;
  if (tid == 0) s_nlist = 0;

  int mode = kModeScan;
  int k = 0;  // sampled keys to reach (0: no sampling, every key is a candidate)
  if (L <= a.budget) {
    mode = kModeAll;
  } else if (L > kExactMax) {
    const double expect = (double)a.budget * kS / (double)L;
    k = (int)ceil(expect + 4.0 * sqrt(expect) + 8.0);
    if (k >= kS / 2) k = 0;
  }
  // decode: the page of the new token (position L - 1), read with the sample's pages
  int32_t st_page = -1;
  if (store) st_page = bt[(L - 1) >> a.page_shift];
  if (k) {
    // the sampled code rows go straight to shared memory with asynchronous 16-byte copies; a
    // warp instruction covers whole groups (kGroup rows of r bytes, one contiguous run when the
    // page holds at least kGroup tokens), so its lanes coalesce into a few line requests. A row
    // on an unusable page is zero-filled and marked invalid.
    constexpr int kPieces = RB / 16;                      // 16-byte pieces per row
    constexpr int kLanesPerGroup = kGroup * kPieces;      // 8 (32-byte rows) or 16 (64-byte)
    constexpr int kGroupsPerIssue = 32 / kLanesPerGroup;  // groups per warp instruction
    constexpr int kWarpGroups = kSampleGroups / kWarps;   // 64 groups per warp
    constexpr int kIssues = kWarpGroups / kGroupsPerIssue;
    const int gl = lane / kLanesPerGroup, piece = lane % kLanesPerGroup;
    const int j = piece / kPieces, part = piece % kPieces;
    int p0[kIssues], pg0[kIssues];
#pragma unroll
    for (int u = 0; u < kIssues; ++u) {
      const int grp = warp * kWarpGroups + u * kGroupsPerIssue + gl;
      p0[u] = sample_group_start(grp, pair, L, kSampleGroups);
      pg0[u] = bt[(p0[u] + (page_size >= kGroup ? 0 : j)) >> a.page_shift];
    }
#pragma unroll
    for (int u = 0; u < kIssues; ++u) {
      const int grp = warp * kWarpGroups + u * kGroupsPerIssue + gl;
      const int pos = p0[u] + j, i = grp * kGroup + j;
      const int32_t pg = (pg0[u] < 0 || (int64_t)pg0[u] >= a.num_pages) ? -1 : pg0[u];
      if (part == 0) sm.valid[i] = pg >= 0;
      const uint8_t* src = a.score_cache +
          ((((int64_t)max(pg, 0) * a.h_kv + h) << a.page_shift) + (pos & (page_size - 1))) * RB;
      cp_async16(smem_u32(sm.rows + i * RB + part * 16), src + part * 16, pg >= 0 ? 16 : 0);
    }
  }
  cp_async_commit();  // (group: the sample rows; M_h is the group before)
  {
    float part[8];
    const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      part[2 * e] = bf16_lo(w[e]);
      part[2 * e + 1] = bf16_hi(w[e]);
    }
    // G > kQGroups (the many heads of a latent layer): batches of kQB rows, their loads issued
    // together, then added in row order
    constexpr int kQB = 16;
#pragma unroll 1
    for (int r0 = rg + kQGroups; rg < kQGroups && r0 < G; r0 += kQB * kQGroups) {
      uint4 v[kQB];
#pragma unroll
      for (int u = 0; u < kQB; ++u) {
        const int r = r0 + u * kQGroups;
        v[u] = r < G ? *reinterpret_cast<const uint4*>(qh + (int64_t)r * D + d8) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kQB; ++u) {
        if (r0 + u * kQGroups >= G) break;
        const uint32_t x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          part[2 * e] += bf16_lo(x[e]);
          part[2 * e + 1] += bf16_hi(x[e]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (rg < kQGroups) sm.qpart[rg][d8 + e] = part[e];
  }
  if (store) {  // decode: copy the new token's K and V rows into the cache
    if (st_page < 0 || (int64_t)st_page >= a.num_pages) {
      if (tid == 0) raise_flag(1u);
      st_page = -1;
    }
    const StoreNew& st = a.store;
    const int pos = L - 1;
#pragma unroll
    for (int u = 0; u < KE; ++u) {
      const int i = tid + u * kThreads;
      if (i >= D) continue;
      s_k[i] = bf16_to_f(k_el[u]);
      if (st_page >= 0) {
        const int64_t base = (int64_t)st_page * st.page_stride +
                             (int64_t)(pos & (page_size - 1)) * st.slot_stride +
                             (int64_t)h * st.head_stride;
        st.k_cache[base + i] = k_el[u];
        if (st.v_cache) st.v_cache[base + i] = v_el[u];
      }
    }
  }
  cp_async_wait<1>();  // M_h landed; the sample rows may still be in flight
  __syncthreads();
  for (int i = tid; i < D; i += kThreads) {
    float acc = 0.f;
    for (int r = 0; r < min(G, kQGroups); ++r) acc += sm.qpart[r][i];
    s_qbar[i] = acc / (float)G;
  }

  __syncthreads();  // qbar

  // ---- p = M_h qbar and, at decode, the new token's code e4m3(M_h k) (or bf16(M_h k)) ----------
  if (!kMSmem) {
    // M_h from global memory: each warp owns kPR / kWarps output rows and reads them together,
    // lanes striding over the projected dimensions (coalesced 128-byte reads, kPR / kWarps
    // independent loads per step), then one warp reduction per row. A latent layer's last 64
    // code columns are its rotary dimensions, passed through (p_j = qbar of that dimension; at
    // decode the code is that dimension of k, rounded once).
    constexpr int kRW = kPR / kWarps;
    static_assert(kPD % 32 == 0 && kPR % kWarps == 0, "projection split");
    if (latent_layer<D>() && tid < R - kPR) {
      const int j = kPR + tid;
      s_p[j] = s_qbar[kPD + tid];
      if (store && st_page >= 0) {
        const int pos = L - 1;
        uint8_t* row = a.store.score_cache +
            (((int64_t)st_page * a.h_kv + h) * page_size + (pos & (page_size - 1))) * RB;
        if (C::kBF16) reinterpret_cast<uint16_t*>(row)[j] = f64_to_bf16((double)s_k[kPD + tid]);
        else row[j] = f64_to_e4m3((double)s_k[kPD + tid]);
      }
    }
    float acc[kRW];
    double acc_k[kRW];
#pragma unroll
    for (int jj = 0; jj < kRW; ++jj) {
      acc[jj] = 0.f;
      acc_k[jj] = 0.0;
    }
    const float* mbase = m_h + (int64_t)(warp * kRW) * kPD;
    static_assert(kPD % 128 == 0, "float4 projection");
    // lane l takes dims 4 l .. 4 l + 3 of every 128-dim span (16-byte loads: the basis is 16-byte
    // aligned, every row starts at a multiple of 512 bytes); two spans' loads in flight together
#pragma unroll 1
    for (int e = 4 * lane; e < kPD; e += 128) {
      const float4 qv = *reinterpret_cast<const float4*>(s_qbar + e);
      double kv[4] = {0.0, 0.0, 0.0, 0.0};
      if (store) {
        const float4 k4 = *reinterpret_cast<const float4*>(s_k + e);
        kv[0] = k4.x; kv[1] = k4.y; kv[2] = k4.z; kv[3] = k4.w;
      }
      float4 mv[kRW];
#pragma unroll
      for (int jj = 0; jj < kRW; ++jj) mv[jj] = __ldg(reinterpret_cast<const float4*>(mbase + jj * kPD + e));
#pragma unroll
      for (int jj = 0; jj < kRW; ++jj) {
        acc[jj] = fmaf(mv[jj].x, qv.x, acc[jj]);
        acc[jj] = fmaf(mv[jj].y, qv.y, acc[jj]);
        acc[jj] = fmaf(mv[jj].z, qv.z, acc[jj]);
        acc[jj] = fmaf(mv[jj].w, qv.w, acc[jj]);
        if (store) {
          acc_k[jj] = fma((double)mv[jj].x, kv[0], acc_k[jj]);
          acc_k[jj] = fma((double)mv[jj].y, kv[1], acc_k[jj]);
          acc_k[jj] = fma((double)mv[jj].z, kv[2], acc_k[jj]);
          acc_k[jj] = fma((double)mv[jj].w, kv[3], acc_k[jj]);
        }
      }
    }
#pragma unroll
    for (int jj = 0; jj < kRW; ++jj) {
      float v = acc[jj];
      double vk = acc_k[jj];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        v += __shfl_xor_sync(0xffffffffu, v, o);
        if (store) vk += __shfl_xor_sync(0xffffffffu, vk, o);
      }
      if (lane == 0) {
        const int j = warp * kRW + jj;
        s_p[j] = v;
        if (store && st_page >= 0) {
          const int pos = L - 1;
          uint8_t* row = a.store.score_cache +
              (((int64_t)st_page * a.h_kv + h) * page_size + (pos & (page_size - 1))) * RB;
          if (C::kBF16) reinterpret_cast<uint16_t*>(row)[j] = f64_to_bf16(vk);
          else row[j] = f64_to_e4m3(vk);
        }
      }
    }
  } else {
    constexpr int TPJ = kThreads / R;  // threads per output
    constexpr int DPT = D / TPJ;
    static_assert(TPJ >= 1 && TPJ <= 32 && D % TPJ == 0, "projection split");
    const int j = tid / TPJ, sub = tid % TPJ;
    const float* mrow = sm.m + j * D;
    float acc = 0.f;
    double acc_k = 0.0;
    // thread sub takes dims sub, sub + TPJ, ... (interleaved: neighbouring threads read
    // neighbouring words)
#pragma unroll
    for (int i = 0; i < DPT; ++i) {
      const int e = i * TPJ + sub;
      acc = fmaf(mrow[e], s_qbar[e], acc);
      if (store) acc_k = fma((double)mrow[e], (double)s_k[e], acc_k);
    }
#pragma unroll
    for (int o = TPJ / 2; o > 0; o >>= 1) {
      acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (store) acc_k += __shfl_xor_sync(0xffffffffu, acc_k, o);
    }
    if (sub == 0) {
      s_p[j] = acc;
      if (store && st_page >= 0) {
        const int pos = L - 1;
        uint8_t* row = a.store.score_cache +
            (((int64_t)st_page * a.h_kv + h) * page_size + (pos & (page_size - 1))) * RB;
        if (C::kBF16) reinterpret_cast<uint16_t*>(row)[j] = f64_to_bf16(acc_k);
        else row[j] = f64_to_e4m3(acc_k);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    // p = 2^-e0 D0 + 2^-e1 D1 (+ ...) with 16-bit digit vectors: D0 = f16(p 2^e0), e0 chosen so
    // that the largest |component| lands in [2^14, 2^15) (inside the f16 range), and D1 =
    // f16(r 2^e1) for the remainder r = p 2^e0 - D0 (exact in fp32), scaled the same way; about
    // 22 significant bits of every component relative to the largest one. BF16 codes multiply
    // bf16 digits (8 significant bits each), four of them for about 24 bits.
    constexpr int kPL = (R + 31) / 32;  // components per lane
    float rem[kPL];
#pragma unroll
    for (int i = 0; i < kPL; ++i) rem[i] = lane + 32 * i < R ? s_p[lane + 32 * i] : 0.f;
    float weight = 1.f;  // 2^-(e0 + ... + e_c): the value of one unit of the current remainder
    for (int c = 0; c < kDigits; ++c) {
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < kPL; ++i) mx = fmaxf(mx, fabsf(rem[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      int ex = 0;
      if (mx > 0.f) ex = min(100, 14 - ((int)((__float_as_uint(mx) >> 23) & 0xFF) - 127));
      const float up = ldexpf(1.0f, ex);
      weight = ldexpf(weight, -ex);
#pragma unroll
      for (int i = 0; i < kPL; ++i) {
        const float v = rem[i] * up;
        const bool in = lane + 32 * i < R;
        if (C::kBF16) {
          const uint16_t db = f_to_bf16(v);
          if (in) s_dig[c * R + lane + 32 * i] = db;
          rem[i] = v - bf16_to_f(db);
        } else {
          const __half dh = __float2half_rn(v);
          if (in) s_dig[c * R + lane + 32 * i] = __half_as_ushort(dh);
          rem[i] = v - __half2float(dh);
        }
      }
      if (lane == 0) s_scale[c] = weight;
    }
  }
  __syncthreads();
  uint8_t* rec = a.prep.rec + (int64_t)pair * kPrepBytes;
  for (int i = tid; i < kDigits * R; i += kThreads) reinterpret_cast<uint16_t*>(rec)[i] = s_dig[i];
  if (tid < kDigits) reinterpret_cast<float*>(rec + kPrepScale)[tid] = s_scale[tid];

  // ---- candidate threshold from the sample ----------------------------------------------------
  uint32_t thr = 0u;       // every key of a finite score is above 0
  uint32_t sample_max = 0u;  // largest sampled key (0: no sample)
  if (k) {
    cp_async_wait<0>();
    __syncthreads();  // every thread's sample rows
    DigitFrags<C> df;
    df.load(s_dig, s_scale, lane);
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    uint32_t key[kTilesPerWarp / 2];  // this lane's sampled keys
#pragma unroll
    for (int u = 0; u < kTilesPerWarp; u += 2) {
      const int i0 = (warp * kTilesPerWarp + u) * 16;
      uint32_t ra0[C::kRegs], rb0[C::kRegs], ra1[C::kRegs], rb1[C::kRegs];
      load_srow<LB>(ra0, sm.rows + (i0 + g) * RB + t * LB);
      load_srow<LB>(rb0, sm.rows + (i0 + g + 8) * RB + t * LB);
      load_srow<LB>(ra1, sm.rows + (i0 + 16 + g) * RB + t * LB);
      load_srow<LB>(rb1, sm.rows + (i0 + 24 + g) * RB + t * LB);
      const float f = pair_scores<C>(ra0, rb0, ra1, rb1, df, t);
      // lane t holds sample 16 * (t >> 1) + 8 * (t & 1) + g of the two tiles
      const int i = i0 + 16 * (t >> 1) + 8 * (t & 1) + g;
      // a sample on an unusable page (flagged by the scan) counts as the lowest key
      key[u / 2] = sm.valid[i] ? score_key(f) : 0u;
      if (key[u / 2] >= 0x00800000u) kmin = min(kmin, key[u / 2]);
      kmax = max(kmax, key[u / 2]);
    }
    block_min_max<kThreads>(kmin, kmax, s_wsum);
    sample_max = kmax;
    // the k-th largest sampled key: the tokens whose keys reach it become candidates
    thr = sample_threshold<kThreads, kSampleBins>(key, (uint32_t)k, kmin, kmax, sm.hist, sm.list,
                                                  &s_nlist, s_wsum, s_info);
  }
  if (tid == 0) {
    *reinterpret_cast<uint32_t*>(rec + kPrepThr) = thr;
    *reinterpret_cast<int*>(rec + kPrepMode) = mode;
    *reinterpret_cast<uint32_t*>(rec + kPrepKmax) = sample_max;
  }
}

// ------------------------------------------------------------------------------------------------
// select
// ------------------------------------------------------------------------------------------------

struct SelectArgs {
  ScanArgs scan;
  int32_t* idx;
  int32_t* count;
};

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelBinBits = 9;  // histogram of the staged candidate keys: 512 bins
constexpr int kSelBins = 1 << kSelBinBits;

constexpr int kSelRun = 12;         // candidates per lane on the flattened register path
constexpr int kSelRegsPerWarp = 8;  // regions per warp on the region-major register path
constexpr int kSelPerRegion = 64;   // entries per region held in registers (two per lane)

// Threshold of the want largest candidate keys held in registers (each(f) calls f(key) for
// every key this thread holds), every key >= base: a histogram in kSelBins bins of 2^hshift
// keys (the top bin also takes every larger key), the bin of the want-th largest key, then the
// exact key by ranking that bin's keys against each other. On return the want largest keys are
// the keys > thr plus the first `take` keys == thr. Returns false when that bin is the top one
// or holds more than 256 keys. s_hist is zero on entry; s_list holds 256 keys.
template <typename EachKey>
__device__ bool threshold_in_registers(EachKey each, uint32_t want, uint32_t base, int hshift,
                                       uint32_t* s_hist, uint32_t* s_list, uint32_t* s_wsum,
                                       int* s_info, int64_t& thr, uint32_t& take) {
  const int tid = threadIdx.x;
  each([&](uint32_t k) {
    atomicAdd(&s_hist[min((uint32_t)kSelBins - 1u, (k - base) >> hshift)], 1u);
  });
  __syncthreads();
  find_bin<kSelThreads>(s_hist, kSelBins, want, s_wsum, s_info);
  const bool found = s_info[3] != 0;
  const uint32_t bin = (uint32_t)s_info[0], m = (uint32_t)s_info[2];
  const uint32_t w2 = want - (uint32_t)s_info[1];
  __syncthreads();  // s_info and s_wsum are rewritten below
  if (!found || bin == kSelBins - 1 || (w2 != m && m > 256)) return false;
  if (w2 == m) {  // the whole bin: every key from its lowest one
    thr = (int64_t)base + ((int64_t)bin << hshift) - 1;
    take = 0;
    return true;
  }
  if (tid == 0) s_info[3] = 0;
  __syncthreads();
  each([&](uint32_t k) {
    if (((k - base) >> hshift) == bin) s_list[atomicAdd(&s_info[3], 1)] = k;
  });
  __syncthreads();
  if (tid < (int)m) {
    const uint32_t x = s_list[tid];
    uint32_t gt = 0, eq = 0;
    for (uint32_t i = 0; i < m; ++i) {
      const uint32_t y = s_list[i];
      gt += y > x;
      eq += y == x;
    }
    if (gt < w2 && w2 <= gt + eq) {  // x is the w2-th largest of the bin (equal keys agree)
      s_info[0] = (int)x;
      s_info[1] = (int)(w2 - gt);
    }
  }
  __syncthreads();
  thr = (int64_t)(uint32_t)s_info[0];
  take = (uint32_t)s_info[1];
  return true;
}

// Warp offsets of the ordered emission: this warp's selected keys come after gt_b keys > thr
// and eq_b keys == thr of the warps before it (s_cnt: 2 kSelWarps words).
__device__ __forceinline__ void warp_offsets(uint32_t n_gt, uint32_t n_eq, uint32_t* s_cnt,
                                             uint32_t& gt_b, uint32_t& eq_b, uint32_t& total_gt,
                                             uint32_t& total_eq) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    s_cnt[warp] = n_gt;
    s_cnt[kSelWarps + warp] = n_eq;
  }
  __syncthreads();
  gt_b = eq_b = total_gt = total_eq = 0u;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    const uint32_t g_ = s_cnt[w], e_ = s_cnt[kSelWarps + w];
    gt_b += w < warp ? g_ : 0u;
    eq_b += w < warp ? e_ : 0u;
    total_gt += g_;
    total_eq += e_;
  }
}

// One ballot group of the ordered emission (32 consecutive candidates, lane order = position
// order): keys > thr, and keys == thr while fewer than `take` came before, go to slot
// (keys > thr before) + min(keys == thr before, take).
__device__ __forceinline__ void emit_group(bool in, int64_t key, int32_t pos, int64_t thr,
                                           uint32_t take, int budget, int32_t* out_idx,
                                           uint32_t& gt_b, uint32_t& eq_b) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const bool is_gt = in && key > thr, is_eq = in && key == thr;
  const unsigned gtm = __ballot_sync(0xffffffffu, is_gt);
  const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
  const uint32_t g_before = gt_b + __popc(gtm & lt), e_before = eq_b + __popc(eqm & lt);
  if (is_gt || (is_eq && e_before < take)) {
    const uint32_t at = g_before + min(e_before, take);
    if (at < (uint32_t)budget) out_idx[at] = pos;
  }
  gt_b += __popc(gtm);
  eq_b += __popc(eqm);
}

__device__ __forceinline__ void select_finish(const SelectArgs& s, int pair, uint32_t want,
                                              uint32_t written, int32_t* out_idx) {
  const int tid = threadIdx.x;
  for (int j = (int)want + tid; j < s.scan.budget; j += kSelThreads) out_idx[j] = -1;
  if (tid == 0) {
    if (written != want) raise_flag(8u);
    s.count[pair] = (int)want;
  }
  // the attention launched next merges its splits through these counters
  clear_attend_tickets(s.scan.cands, pair);
}

// Region-major register path (at most kSelWarps * kSelRegsPerWarp regions): warp w holds
// regions [w kSelRegsPerWarp, (w + 1) kSelRegsPerWarp), lane l entries l and l + 32 of each,
// loaded together with the region counts (one round trip, no offsets needed: the warp's
// candidates are in position order). Returns false, having written nothing, when a region holds
// more than kSelPerRegion candidates, there are fewer candidates than wanted, or the threshold
// bin cannot be resolved (s_hist is then dirty).
__device__ bool select_region_major(const SelectArgs& s, int pair, int n_reg, int seg,
                                    uint32_t want, uint32_t base, int hshift, uint32_t* s_hist,
                                    uint32_t* s_list, uint32_t* s_wsum, uint32_t* s_cnt,
                                    int* s_info) {
  constexpr int RW = kSelRegsPerWarp, E = kSelPerRegion / 32;
  const ScanArgs& a = s.scan;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t* ck = a.cands.key + (int64_t)pair * n_reg * seg;
  const int32_t* cp = a.cands.pos + (int64_t)pair * n_reg * seg;
  const uint32_t* cc = a.cands.cnt + (int64_t)pair * n_reg;
  uint32_t cnt[RW], key[RW][E];
  int32_t pos[RW][E];
#pragma unroll
  for (int u = 0; u < RW; ++u) {
    const int r = warp * RW + u;
    cnt[u] = r < n_reg ? cc[r] : 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      key[u][e] = r < n_reg ? ck[(int64_t)r * seg + lane + 32 * e] : 0u;
      pos[u][e] = r < n_reg ? cp[(int64_t)r * seg + lane + 32 * e] : 0;
    }
  }
  uint32_t wn = 0, over = 0;
#pragma unroll
  for (int u = 0; u < RW; ++u) {
    wn += cnt[u];
    over |= cnt[u] > (uint32_t)kSelPerRegion;
  }
  if (lane == 0) {
    s_cnt[warp] = wn;
    s_cnt[kSelWarps + warp] = over;
  }
  __syncthreads();
  uint32_t n = 0;
  over = 0;
#pragma unroll
  for (int w = 0; w < kSelWarps; ++w) {
    n += s_cnt[w];
    over |= s_cnt[kSelWarps + w];
  }
  __syncthreads();  // s_cnt is rewritten below
  if (over || n < want) return false;
  auto each = [&](auto&& f) {
#pragma unroll
    for (int u = 0; u < RW; ++u)
#pragma unroll
      for (int e = 0; e < E; ++e)
        if ((uint32_t)(lane + 32 * e) < cnt[u]) f(key[u][e]);
  };
  int64_t thr;
  uint32_t take;
  if (!threshold_in_registers(each, want, base, hshift, s_hist, s_list, s_wsum, s_info, thr, take))
    return false;
  uint32_t n_gt = 0, n_eq = 0;
  each([&](uint32_t k) {
    n_gt += (int64_t)k > thr;
    n_eq += (int64_t)k == thr;
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
    n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
  }
  uint32_t gt_b, eq_b, total_gt, total_eq;
  warp_offsets(n_gt, n_eq, s_cnt, gt_b, eq_b, total_gt, total_eq);
  int32_t* out_idx = s.idx + (int64_t)pair * a.budget;
#pragma unroll
  for (int u = 0; u < RW; ++u)
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (32 * e < (int)cnt[u])  // (warp-uniform)
        emit_group((uint32_t)(lane + 32 * e) < cnt[u], key[u][e], pos[u][e], thr, take, a.budget,
                   out_idx, gt_b, eq_b);
  select_finish(s, pair, want, total_gt + min(total_eq, take), out_idx);
  return true;
}

// Flattened register path (at most kSelThreads * kSelRun candidates, any region count, offsets
// s_roff known): warp w owns a contiguous span of 32 kSelRun candidates at most, lane l the
// candidates span + 32 u + l (coalesced loads straight from the regions). Returns false, having
// written nothing, when the threshold bin cannot be resolved (s_hist is then dirty).
template <typename RegionOf>
__device__ bool select_in_registers(const SelectArgs& s, int pair, int n_reg, int seg,
                                    uint32_t want, uint32_t base, int hshift, RegionOf region_of,
                                    const uint32_t* s_roff, uint32_t* s_hist, uint32_t* s_list,
                                    uint32_t* s_wsum, uint32_t* s_cnt, int* s_info) {
  const ScanArgs& a = s.scan;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = (int)s_roff[n_reg];
  const uint32_t* ck = a.cands.key + (int64_t)pair * n_reg * seg;
  const int32_t* cp = a.cands.pos + (int64_t)pair * n_reg * seg;
  const int span = ((n + kSelWarps - 1) / kSelWarps + 31) & ~31;  // <= 32 kSelRun
  const int lo = min(n, warp * span), hi = min(n, lo + span);
  uint32_t key[kSelRun];
  int32_t pos[kSelRun];
  int r = lo + lane < hi ? region_of(lo + lane) : 0;
#pragma unroll
  for (int u = 0; u < kSelRun; ++u) {
    const int j = lo + 32 * u + lane;
    key[u] = 0u;
    pos[u] = 0;
    if (j < hi) {
      while (s_roff[r + 1] <= (uint32_t)j) ++r;
      const int64_t src = (int64_t)r * seg + (j - (int)s_roff[r]);
      key[u] = ck[src];
      pos[u] = cp[src];
    }
  }
  auto each = [&](auto&& f) {
#pragma unroll
    for (int u = 0; u < kSelRun; ++u)
      if (lo + 32 * u + lane < hi) f(key[u]);
  };
  int64_t thr;
  uint32_t take;
  if (!threshold_in_registers(each, want, base, hshift, s_hist, s_list, s_wsum, s_info, thr, take))
    return false;
  uint32_t n_gt = 0, n_eq = 0;
  each([&](uint32_t k) {
    n_gt += (int64_t)k > thr;
    n_eq += (int64_t)k == thr;
  });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
    n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
  }
  uint32_t gt_b, eq_b, total_gt, total_eq;
  warp_offsets(n_gt, n_eq, s_cnt, gt_b, eq_b, total_gt, total_eq);
  int32_t* out_idx = s.idx + (int64_t)pair * a.budget;
#pragma unroll
  for (int u = 0; u < kSelRun; ++u)
    if (lo + 32 * u < hi)  // (warp-uniform)
      emit_group(lo + 32 * u + lane < hi, key[u], pos[u], thr, take, a.budget, out_idx, gt_b,
                 eq_b);
  select_finish(s, pair, want, total_gt + min(total_eq, take), out_idx);
  return true;
}

template <int D, class C>
__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs s) {
  extern __shared__ uint32_t sel_dyn[];  // keys [kSelectCap] then positions [kSelectCap]
  uint32_t* s_ckey = sel_dyn;
  int32_t* s_cpos = reinterpret_cast<int32_t*>(sel_dyn + kSelectCap);
  __shared__ uint32_t s_hist[kBins];
  __shared__ int s_info[4];
  __shared__ uint32_t s_roff[kMaxRegions + 1];
  __shared__ uint32_t s_wsum[2 * kSelWarps];
  __shared__ uint64_t s_red64[kSelWarps];

  const ScanArgs& a = s.scan;
  const int tid = threadIdx.x, lane = tid & 31;
  const int pair = blockIdx.x;
  const int b = pair / a.h_kv;
  const int L = clamp_len(a.seq_lens[b], a.max_pages << a.page_shift);
  const int budget = a.budget;
  int32_t* out_idx = s.idx + (int64_t)pair * budget;
  // the prep's record: the prep grid completed before any scan CTA passed its own wait, and
  // this grid starts only once every scan CTA has passed it, so the record may be read before
  // waiting for the scan (from L2: no stale L1 line)
  const uint8_t* rec = a.prep.rec + (int64_t)pair * kPrepBytes;
  const int mode = __ldcg(reinterpret_cast<const int*>(rec + kPrepMode));
  const uint32_t base = __ldcg(reinterpret_cast<const unsigned int*>(rec + kPrepThr));
  const uint32_t sample_max = __ldcg(reinterpret_cast<const unsigned int*>(rec + kPrepKmax));
  pdl_wait();  // the scan's candidates
  pdl_trigger();  // the attention may be scheduled; it waits for this grid to complete
  if (mode == kModeAll) {
    for (int j = tid; j < budget; j += kSelThreads) out_idx[j] = j < L ? j : -1;
    if (tid == 0) s.count[pair] = L;
    clear_attend_tickets(a.cands, pair);
    return;
  }
  const int n_reg = a.n_chunks * kRegionsPerChunk;
  const int seg = a.chunk / kRegionsPerChunk;
  const uint32_t* ck = a.cands.key + (int64_t)pair * n_reg * seg;
  const int32_t* cp = a.cands.pos + (int64_t)pair * n_reg * seg;
  const uint32_t* cc = a.cands.cnt + (int64_t)pair * n_reg;
  const uint32_t want = (uint32_t)min(budget, L);
  // histogram of the candidate keys over [the prep's threshold, the largest sampled key] (keys
  // above it fall into the top bin)
  bool use_hist = base > 0u && sample_max > base;
  const int hshift = use_hist ? max(0, (32 - __clz(sample_max - base)) - kSelBinBits) : 0;
  for (int i = tid; i < kSelBins; i += kSelThreads) s_hist[i] = 0u;
  uint32_t* s_cnt = reinterpret_cast<uint32_t*>(s_red64);  // 2 kSelWarps words
  if (use_hist && n_reg <= kSelWarps * kSelRegsPerWarp) {
    if (select_region_major(s, pair, n_reg, seg, want, base, hshift, s_hist, s_ckey, s_wsum,
                            s_cnt, s_info))
      return;
    __syncthreads();
    for (int i = tid; i < kSelBins; i += kSelThreads) s_hist[i] = 0u;  // (paths below)
  }

  // region offsets: exclusive prefix of the counts, in position order (each thread loads and
  // sums a run of adjacent regions, then a block-wide scan)
  auto offsets = [&]() {
    constexpr int kPer = kMaxRegions / kSelThreads;
    const int per = (n_reg + kSelThreads - 1) / kSelThreads;  // <= kPer
    const int r0 = min(n_reg, tid * per), r1 = min(n_reg, r0 + per);
    uint32_t v[kPer];
    uint32_t sum = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      v[i] = r0 + i < r1 ? cc[r0 + i] : 0u;
      sum += v[i];
    }
    uint64_t total;
    uint32_t run = (uint32_t)block_excl_scan64<kSelThreads>(sum, total, s_red64);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (r0 + i < r1) s_roff[r0 + i] = run;
      run += v[i];
    }
    if (tid == 0) s_roff[n_reg] = (uint32_t)total;
    __syncthreads();
  };
  offsets();
  // flattened candidate j -> region (the last r with s_roff[r] <= j)
  auto region_of = [&](int j) {
    int lo = 0, hi = n_reg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_roff[mid] <= (uint32_t)j) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  if (use_hist && s_roff[n_reg] >= want && s_roff[n_reg] <= (uint32_t)(kSelThreads * kSelRun)) {
    if (select_in_registers(s, pair, n_reg, seg, want, base, hshift, region_of, s_roff, s_hist,
                            s_ckey, s_wsum, s_cnt, s_info))
      return;
    for (int i = tid; i < kSelBins; i += kSelThreads) s_hist[i] = 0u;  // (general path below)
    __syncthreads();
  }
  if (s_roff[n_reg] < want) {
    // rescue: the sampled threshold was too high; score every token of the sequence again with
    // no threshold (all keys become candidates), then select exactly as usual
    if (tid == 0) raise_flag(16u);
    use_hist = false;
    DigitFrags<C> df;
    df.load(reinterpret_cast<const uint16_t*>(rec), reinterpret_cast<const float*>(rec + kPrepScale),
            lane);
    int32_t* s_page = reinterpret_cast<int32_t*>(s_ckey);  // free until the staging below
    for (int c = 0; c < a.n_chunks; ++c) {
      const int start = c * a.chunk;
      const int n_local = max(0, min(a.chunk, L - start));
      const int n_pages = (n_local + (1 << a.page_shift) - 1) >> a.page_shift;
      __syncthreads();
      load_pages(s_page, a.block_table + (int64_t)b * a.max_pages + (start >> a.page_shift),
                 n_pages, a.num_pages);
      __syncthreads();
      scan_chunk<C, false>(a, pair, c, L, 0u, df, s_page, nullptr);
    }
    __syncthreads();
    offsets();
  }
  const uint32_t n = s_roff[n_reg];
  const bool staged = n <= (uint32_t)kSelectCap;
  auto src_of = [&](int j) -> int64_t {
    const int r = region_of(j);
    return (int64_t)r * seg + (j - (int)s_roff[r]);
  };
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  if (staged) {
    // flatten the regions (keys and positions, position order) into shared memory: each warp
    // copies 8 regions at a time, the first 64 candidates of each with all loads issued before
    // any store (one round trip), the rare rest of a longer region afterwards; key range and
    // histogram on the way
    auto put = [&](uint32_t at, uint32_t key, int32_t pos) {
      s_ckey[at] = key;
      s_cpos[at] = pos;
      kmin = min(kmin, key);
      kmax = max(kmax, key);
      if (use_hist) atomicAdd(&s_hist[min((uint32_t)kSelBins - 1u, (key - base) >> hshift)], 1u);
    };
    constexpr int kRB = 8;
    for (int rb = (tid >> 5) * kRB; rb < n_reg; rb += kSelWarps * kRB) {
      uint32_t kk[kRB][2];
      int32_t pp[kRB][2];
#pragma unroll
      for (int u = 0; u < kRB; ++u) {
        const int r = rb + u;
        const uint32_t cnt = r < n_reg ? s_roff[r + 1] - s_roff[r] : 0u;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t i = lane + 32 * e;
          kk[u][e] = i < cnt ? ck[(int64_t)r * seg + i] : 0u;
          pp[u][e] = i < cnt ? cp[(int64_t)r * seg + i] : 0;
        }
      }
#pragma unroll
      for (int u = 0; u < kRB; ++u) {
        const int r = rb + u;
        const uint32_t cnt = r < n_reg ? s_roff[r + 1] - s_roff[r] : 0u;
        const uint32_t off = r < n_reg ? s_roff[r] : 0u;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t i = lane + 32 * e;
          if (i < cnt) put(off + i, kk[u][e], pp[u][e]);
        }
        for (uint32_t i = 64 + lane; i < cnt; i += 32)
          put(off + i, ck[(int64_t)r * seg + i], cp[(int64_t)r * seg + i]);
      }
    }
  } else {
    for (int j = tid; j < (int)n; j += kSelThreads) {
      const uint32_t key = ck[src_of(j)];
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
  }
  __syncthreads();  // the staged candidates and their histogram
  auto key_at = [&](int j) -> uint32_t { return staged ? s_ckey[j] : ck[src_of(j)]; };
  auto pos_at = [&](int j) -> int32_t { return staged ? s_cpos[j] : cp[src_of(j)]; };
  int64_t thr;
  uint32_t take;
  const bool done = use_hist && staged &&
                    threshold_from_hist<kSelThreads, kSelBins>(key_at, (int)n, want, base, hshift,
                                                               s_hist, s_wsum, s_info, thr, take);
  if (!done) {
    block_min_max<kSelThreads>(kmin, kmax, s_wsum);
    select_threshold<kSelThreads>(key_at, (int)n, want, kmin, kmax, s_hist, s_wsum, s_info, thr,
                                  take);
  }
  // ordered emission: the selected candidates are the keys > thr and the first `take` keys == thr
  // in position order; candidate j goes to slot (keys > thr before it) + min(keys == thr before
  // it, take). Thread i owns the contiguous run [i q, i q + q) of candidates (q a multiple of 4:
  // 16-byte shared loads when staged); one block-wide scan of its two counts gives its offsets.
  const int q = (((int)n + kSelThreads - 1) / kSelThreads + 3) & ~3;
  const int lo = min((int)n, tid * q), hi = min((int)n, lo + q);
  uint32_t n_gt = 0, n_eq = 0;
  if (staged) {
    for (int j0 = lo; j0 < hi; j0 += 4) {
      const uint4 k4 = *reinterpret_cast<const uint4*>(s_ckey + j0);
      const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool in = j0 + e < hi;
        n_gt += in && (int64_t)kv[e] > thr;
        n_eq += in && (int64_t)kv[e] == thr;
      }
    }
  } else {
    for (int j = lo; j < hi; ++j) {
      const int64_t key = key_at(j);
      n_gt += key > thr;
      n_eq += key == thr;
    }
  }
  uint64_t totals;
  const uint64_t before =
      block_excl_scan64<kSelThreads>(((uint64_t)n_gt << 32) | n_eq, totals, s_red64);
  const uint32_t total_gt = (uint32_t)(totals >> 32), total_eq = (uint32_t)totals;
  uint32_t gt_b = (uint32_t)(before >> 32), eq_b = (uint32_t)before;
  auto emit = [&](int64_t key, int j) {
    if (key > thr) {
      const uint32_t at = gt_b + min(eq_b, take);
      if (at < (uint32_t)budget) out_idx[at] = pos_at(j);
      ++gt_b;
    } else if (key == thr) {
      if (eq_b < take && gt_b + eq_b < (uint32_t)budget) out_idx[gt_b + eq_b] = pos_at(j);
      ++eq_b;
    }
  };
  if (staged) {
    for (int j0 = lo; j0 < hi; j0 += 4) {
      const uint4 k4 = *reinterpret_cast<const uint4*>(s_ckey + j0);
      const uint32_t kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (j0 + e < hi) emit((int64_t)kv[e], j0 + e);
    }
  } else {
    for (int j = lo; j < hi; ++j) emit((int64_t)key_at(j), j);
  }
  const uint32_t written = total_gt + min(total_eq, take);
  for (int j = (int)want + tid; j < budget; j += kSelThreads) out_idx[j] = -1;
  if (tid == 0) {
    if (written != want) raise_flag(8u);
    s.count[pair] = (int)want;
  }
  // the attention launched next merges its splits through these counters
  clear_attend_tickets(a.cands, pair);
}

template <typename Kern, typename... Args>
cudaError_t launch_k(Kern kern, dim3 grid, int threads, size_t smem, bool pdl, cudaStream_t s,
                     const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, class C>
cudaError_t launch_t(const ScorePlan& plan, int pairs, const PrepArgs& pa, const ScanArgs& sa,
                     const SelectArgs& sel, bool store, bool pdl, cudaStream_t s) {
  cudaError_t e;
  const size_t prep_smem = sizeof(PrepSmem<D, C>);
  if (store) {
    // (the fused decode store exists for the head dimensions that have decode attention: the GQA
    // layers and the latent rows of multi-head latent attention)
    if constexpr (D == 128 || D == 256 || D == 576) {
      e = configure_kernel((const void*)prep_kernel<D, C, true>, (int)prep_smem, false);
      if (e == cudaSuccess)
        e = launch_k(prep_kernel<D, C, true>, dim3(pairs), kThreads, prep_smem, pdl, s, pa);
    } else {
      e = cudaErrorInvalidValue;
    }
  } else {
    e = configure_kernel((const void*)prep_kernel<D, C, false>, (int)prep_smem, false);
    if (e == cudaSuccess)
      e = launch_k(prep_kernel<D, C, false>, dim3(pairs), kThreads, prep_smem, pdl, s, pa);
  }
  if (e != cudaSuccess) return e;
  const size_t scan_smem =
      (size_t)scan_ring_bytes<C>() + (size_t)(plan.chunk / (1 << sa.page_shift) + 1) * 4;
  e = configure_kernel((const void*)scan_kernel<D, C>, (int)scan_smem, false);
  if (e != cudaSuccess) return e;
  e = launch_k(scan_kernel<D, C>, dim3(plan.n_chunks, pairs), kThreads, scan_smem, true, s, sa);
  if (e != cudaSuccess) return e;
  const size_t sel_smem = (size_t)kSelectCap * 8;
  e = configure_kernel((const void*)select_kernel<D, C>, (int)sel_smem, false);
  if (e != cudaSuccess) return e;
  return launch_k(select_kernel<D, C>, dim3(pairs), kSelThreads, sel_smem, true, s, sel);
}

}  // namespace score_detail

ScorePlan plan_score(int pairs, int max_seq_len, int page_size, int d) {
  using namespace score_detail;
  ScorePlan p;
  // positions per scan CTA: a power of two in [2048, 8192] and a multiple of the page size,
  // smaller while the grid would not cover every SM several times over, as long as a pair's
  // candidate regions stay within what the select handles cheaply: the region-major register
  // tier, or twice that for d = 128 (16- to 64-byte scoring rows, where a scan CTA is short and
  // the flattened register tier costs less than the SMs the scan would leave idle; measured at
  // 128K context, 1 and 4 sequences). With few pairs and long contexts the select, one CTA per
  // pair, would otherwise cost more than the scan saves.
  const long long region_cap = (d == 128 ? 2LL : 1LL) * kSelWarps * kSelRegsPerWarp;
  int chunk = 8192;
  while (chunk > 2048 &&
         (long long)pairs * ((max_seq_len + chunk - 1) / chunk) < 6LL * num_sms() &&
         (long long)((max_seq_len + chunk / 2 - 1) / (chunk / 2)) * kRegionsPerChunk <= region_cap)
    chunk >>= 1;
  while (chunk % page_size) chunk <<= 1;
  while ((long long)((max_seq_len + chunk - 1) / chunk) * kRegionsPerChunk > kMaxRegions) chunk <<= 1;
  p.chunk = chunk;
  p.n_chunks = (max_seq_len + chunk - 1) / chunk;
  if (p.n_chunks < 1) p.n_chunks = 1;
  const size_t prep = (size_t)pairs * kPrepBytes;
  const size_t counts = ((size_t)pairs * p.n_chunks * kRegionsPerChunk * 4 + 255) / 256 * 256;
  const size_t entries = (size_t)pairs * p.n_chunks * chunk;
  p.ws_bytes = prep + counts + entries * 8;
  return p;
}

cudaError_t launch_score_topk(const uint16_t* q, const float* basis, const uint8_t* score_cache,
                              const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                              int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                              int page_size, int budget, int32_t* idx, int32_t* count, void* ws,
                              int* attend_tickets, const StoreNew* store, bool pdl,
                              cudaStream_t s, bool bf16_codes, int tickets_per_pair) {
  using namespace score_detail;
  const int pairs = batch * h_kv;
  if (pairs == 0) return cudaSuccess;
  const ScorePlan plan = plan_score(pairs, max_pages * page_size, page_size, d);
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const Prep prep{w};
  const size_t counts = ((size_t)pairs * plan.n_chunks * kRegionsPerChunk * 4 + 255) / 256 * 256;
  const size_t entries = (size_t)pairs * plan.n_chunks * plan.chunk;
  Cands cands;
  cands.cnt = reinterpret_cast<uint32_t*>(w + (size_t)pairs * kPrepBytes);
  cands.key = reinterpret_cast<uint32_t*>(w + (size_t)pairs * kPrepBytes + counts);
  cands.pos = reinterpret_cast<int32_t*>(w + (size_t)pairs * kPrepBytes + counts + entries * 4);
  cands.attend_tickets = attend_tickets;
  cands.tickets_per_pair = tickets_per_pair;

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
  const bool st = store != nullptr;
  if (bf16_codes) {
    if (d == 128 && r == 32)
      return launch_t<128, Codes<32, true>>(plan, pairs, pa, sa, sel, st, pdl, s);
    return cudaErrorInvalidValue;
  }
  if (d == 128 && r == 16) return launch_t<128, Codes<16, false>>(plan, pairs, pa, sa, sel, st, pdl, s);
  if (d == 128 && r == 32) return launch_t<128, Codes<32, false>>(plan, pairs, pa, sa, sel, st, pdl, s);
  if (d == 128 && r == 64) return launch_t<128, Codes<64, false>>(plan, pairs, pa, sa, sel, st, pdl, s);
  if (d == 256 && r == 64) return launch_t<256, Codes<64, false>>(plan, pairs, pa, sa, sel, st, pdl, s);
  // multi-head latent attention: basis rank r over the 512 latent dimensions, r + 64 code columns
  if (d == 576 && r == 64) return launch_t<576, Codes<128, false>>(plan, pairs, pa, sa, sel, st, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
