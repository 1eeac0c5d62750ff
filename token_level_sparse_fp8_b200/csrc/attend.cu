// Gather-free indexed attention and the dense paged decode baseline (JSSA summary, section 3.1
// step 3 and section 3.3; JSSA README, section 3 microbenchmark against full-KV decode).
//
// Grid: (splits, batch * h_kv). A CTA owns one (sequence b, KV head h) and one contiguous range
// of its positions -- a slice of the index set (indexed mode) or of [lo, seq_len) (dense mode).
//   * Row addresses: the CTA first turns each of its positions into a 64-bit element offset
//     (page-table lookup, bounds checked) kept in shared memory.
//   * Each of the 4 warps walks its own 16-token tiles. A tile's K and V rows (2d bytes each:
//     256 B at d = 128, 512 B at d = 256) are copied straight from their paged locations into the warp's ring of kStages
//     shared-memory stages with 16-byte cp.async (rows past the slice or on unusable pages are
//     zero-filled) -- no staging buffer in global memory -- so kStages - 1 tiles are in flight
//     while one is computed. Inside a stage a row's 16-byte chunk c sits at chunk c ^ (row & 7),
//     which makes the ldmatrix reads below conflict-free.
//   * Tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate) with the 16 tokens as the M
//     rows and the G <= 8 query heads of the KV head as the N columns: S^T = K Q^T (K fragments
//     by ldmatrix), then O^T += V^T P^T (V^T fragments by ldmatrix.trans). P^T reaches the
//     B-operand layout with movmatrix, split into a bf16 high and low part so the probabilities
//     keep ~16 significant bits.
//   * Online softmax in the log2 domain; warps merge in shared memory; CTAs of one (b, h) merge
//     through fp32 partials (m, l, o) in the workspace, the last CTA to take the ticket combines
//     them, writes the bf16 output and resets the ticket.
#include <float.h>

#include "common.cuh"

namespace jssa {

namespace attend_detail {

constexpr int kWarps = kAttendWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = kAttendTile;
constexpr int kMaxChunk = 1024;  // positions per CTA (row offsets kept in shared memory)
constexpr int kStages = 3;       // tiles per warp ring (kStages - 1 in flight)
// Shared-memory ring geometry for head dim D: K (or V) rows of one tile, a stage (K then V), the
// dynamic shared memory of a CTA; CTAs per SM (d = 128: two; d = 256: one, its ring is 192 KB).
template <int D>
struct Ring {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kChunks = kRowBytes / 16;  // 16-byte chunks per row
  static constexpr int kTileBytes = kTile * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kBytes = kWarps * kStages * kStageBytes;
  static constexpr int kCtasPerSm = D == 128 ? 2 : 1;
};

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

template <int D, bool INDEXED>
__global__ void __launch_bounds__(kThreads, Ring<D>::kCtasPerSm)
    attend_kernel(AttendArgs a, int chunk, int splits) {
  static_assert(D == 128 || D == 256, "head dim");
  constexpr int KB = D / 16;  // k-blocks of S^T, m-tiles of O^T
  constexpr int kRowBytes = Ring<D>::kRowBytes, kChunks = Ring<D>::kChunks;
  constexpr int kTileBytes = Ring<D>::kTileBytes, kStageBytes = Ring<D>::kStageBytes;
  extern __shared__ __align__(128) uint8_t att_ring[];  // warp rings; the warp merge reuses it
  __shared__ int64_t s_off[kMaxChunk];
  __shared__ float s_m[kWarps][kAttendMaxG], s_l[kWarps][kAttendMaxG];
  __shared__ int s_last;
  float(*s_o)[kAttendMaxG][D] = reinterpret_cast<float(*)[kAttendMaxG][D]>(att_ring);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int pair = blockIdx.y, split = blockIdx.x;
  const int b = pair / a.h_kv, h = pair % a.h_kv;
  const int G = a.h_q / a.h_kv;
  const int max_len = a.max_pages * a.page_size;

  // dense mode: launched as a programmatic dependent of whatever precedes it on the stream, so
  // nothing (queries, lengths, caches) is read before that kernel has completed; the launch itself
  // overlaps the previous kernel's tail
  if (!INDEXED) pdl_wait();
  // Q^T fragments (B operand of S^T = K Q^T): column n = head g of this KV head (zero for g >= G);
  // k-block kb: dims 16kb + 2t, +1 (b0) and 16kb + 8 + 2t, +1 (b1)
  uint32_t qb0[KB], qb1[KB];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        a.q + ((int64_t)b * a.h_q + (int64_t)h * G + (g < G ? g : 0)) * D);
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
      qb0[kb] = g < G ? qrow[8 * kb + t] : 0u;
      qb1[kb] = g < G ? qrow[8 * kb + 4 + t] : 0u;
    }
  }

  int n_total, lo = 0;
  if (INDEXED) {
    pdl_wait();  // index sets come from the preceding score + top-B kernel
    n_total = a.count[pair];
    n_total = n_total < 0 ? 0 : (n_total > a.budget ? a.budget : n_total);
  } else {
    int L = a.seq_lens[b];
    if (L < 0 || L > max_len) {
      if (tid == 0 && split == 0) raise_flag(4u);
      L = L < 0 ? 0 : max_len;
    }
    lo = a.window > 0 ? max(0, L - a.window) : 0;
    n_total = L - lo;
  }
  const int j_begin = split * chunk;
  const int n_mine = max(0, min(chunk, n_total - j_begin));

  // ---- row offsets of this CTA's positions: all index loads, then all page-table loads -------
  {
    constexpr int kPer = kMaxChunk / kThreads;
    const int32_t* bt = a.block_table + (int64_t)b * a.max_pages;
    int pos[kPer], pg[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int j = tid + u * kThreads;
      pos[u] = -1;
      if (j < n_mine)
        pos[u] = INDEXED ? a.idx[(int64_t)pair * a.budget + j_begin + j] : lo + j_begin + j;
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
      else
        off = (int64_t)pg[u] * a.page_stride + (int64_t)(pos[u] % a.page_size) * a.slot_stride +
              (int64_t)h * a.head_stride;
      s_off[j] = off;
    }
  }
  __syncthreads();
  // a kernel launched next may be scheduled now; it waits for this grid to complete before
  // reading anything (the decode step's first kernel does)
  pdl_trigger();

  // ---- per-warp tiles through a ring of shared-memory stages --------------------------------
  const int n_tiles = (n_mine + kTile - 1) / kTile;
  const int n_warp_tiles = warp < n_tiles ? (n_tiles - warp + kWarps - 1) / kWarps : 0;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  float o[KB][4];
#pragma unroll
  for (int m = 0; m < KB; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // heads 2t, 2t+1

  const uint32_t ring = smem_u32(att_ring) + warp * kStages * kStageBytes;
  // copies of tile `tl` into stage `st`: piece p = 32 it + lane is row p / kChunks, chunk
  // p % kChunks
  auto issue = [&](int tl, int st) {
    const int j0 = tl * kTile;
#pragma unroll
    for (int it = 0; it < kTile * kChunks / 32; ++it) {
      const int p = 32 * it + lane;
      const int row = p / kChunks, c = p % kChunks;
      const int j = j0 + row;
      const int64_t off = j < n_mine ? s_off[j] : -1;
      const int64_t src = (off >= 0 ? off : 0) + c * 8;
      const uint32_t dst = ring + st * kStageBytes + row * kRowBytes + ((c ^ (row & 7)) << 4);
      cp_async16(dst, a.k_cache + src, off >= 0 ? 16 : 0);
      cp_async16(dst + kTileBytes, a.v_cache + src, off >= 0 ? 16 : 0);
    }
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < n_warp_tiles) issue(warp + kWarps * i, i);
    cp_async_commit();
  }
  // ldmatrix row addresses (lane -> matrix lane / 8, row lane % 8)
  const int mat = lane >> 3, mr = lane & 7;
  const int k_row = (mat & 1) * 8 + mr, k_half = mat >> 1;  // K: rows 0-7 / 8-15, k lo / hi
  const int v_row = (mat >> 1) * 8 + mr, v_half = mat & 1;  // V: tokens 0-7 / 8-15, dims lo / hi
  for (int i = 0; i < n_warp_tiles; ++i) {
    if (i + kStages - 1 < n_warp_tiles)
      issue(warp + kWarps * (i + kStages - 1), (i + kStages - 1) % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const int tile = warp + kWarps * i;
    const uint32_t st = ring + (i % kStages) * kStageBytes;

    // S^T (16 tokens x 8 heads) = K Q^T
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
      const int c = 2 * kb + k_half;
      uint32_t a0, a1, a2, a3;
      ldsm_x4(st + k_row * kRowBytes + ((c ^ (k_row & 7)) << 4), a0, a1, a2, a3);
      mma_bf16(s, a0, a1, a2, a3, qb0[kb], qb1[kb]);
    }
    // rows: token g (s[0], s[1]) and g+8 (s[2], s[3]); columns: heads 2t, 2t+1
    const int j0 = tile * kTile;
    const bool ok0 = j0 + g < n_mine && s_off[j0 + g] >= 0;
    const bool ok1 = j0 + g + 8 < n_mine && s_off[j0 + g + 8] >= 0;
    float x[4];
    x[0] = ok0 ? s[0] * scale_log2 : -INFINITY;
    x[1] = ok0 ? s[1] * scale_log2 : -INFINITY;
    x[2] = ok1 ? s[2] * scale_log2 : -INFINITY;
    x[3] = ok1 ? s[3] * scale_log2 : -INFINITY;
    float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
    for (int sh = 4; sh < 32; sh <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, sh));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, sh));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float corr0 = fast_exp2(m_run[0] - mu0), corr1 = fast_exp2(m_run[1] - mu1);
    float p[4];
    p[0] = fast_exp2(x[0] - mu0);
    p[1] = fast_exp2(x[1] - mu1);
    p[2] = fast_exp2(x[2] - mu0);
    p[3] = fast_exp2(x[3] - mu1);
    l_run[0] = l_run[0] * corr0 + p[0] + p[2];
    l_run[1] = l_run[1] * corr1 + p[1] + p[3];
    m_run[0] = mn0;
    m_run[1] = mn1;
#pragma unroll
    for (int m = 0; m < KB; ++m) {
      o[m][0] *= corr0;
      o[m][1] *= corr1;
      o[m][2] *= corr0;
      o[m][3] *= corr1;
    }
    // P^T as the B operand (tokens x heads), high and low bf16 parts
    const uint32_t ph0 = pack_bf16x2(p[0], p[1]);  // token g,   heads 2t, 2t+1
    const uint32_t ph1 = pack_bf16x2(p[2], p[3]);  // token g+8
    const uint32_t pl0 = pack_bf16x2(p[0] - bf16_lo(ph0), p[1] - bf16_hi(ph0));
    const uint32_t pl1 = pack_bf16x2(p[2] - bf16_lo(ph1), p[3] - bf16_hi(ph1));
    const uint32_t bh0 = movmatrix_t(ph0), bh1 = movmatrix_t(ph1);
    const uint32_t bl0 = movmatrix_t(pl0), bl1 = movmatrix_t(pl1);
    // O^T (dims x heads) += V^T P^T; m-tile m: rows = dims 16m + g and 16m + g + 8
#pragma unroll
    for (int m = 0; m < KB; ++m) {
      const int c = 2 * m + v_half;
      uint32_t va0, va1, va2, va3;
      ldsm_x4_t(st + kTileBytes + v_row * kRowBytes + ((c ^ (v_row & 7)) << 4), va0, va1, va2,
                va3);
      mma_bf16(o[m], va0, va1, va2, va3, bh0, bh1);
      mma_bf16(o[m], va0, va1, va2, va3, bl0, bl1);
    }
    __syncwarp();  // the stage is refilled by the next iteration's copies
  }
  cp_async_wait<0>();
#pragma unroll
  for (int sh = 4; sh < 32; sh <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], sh);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], sh);
  }

  // ---- merge the 4 warps (their rings are done: the shared memory is reused) ------------------
  __syncthreads();
  {
    const int hh0 = 2 * t, hh1 = 2 * t + 1;
    if (g == 0) {
      if (hh0 < G) { s_m[warp][hh0] = m_run[0]; s_l[warp][hh0] = l_run[0]; }
      if (hh1 < G) { s_m[warp][hh1] = m_run[1]; s_l[warp][hh1] = l_run[1]; }
    }
#pragma unroll
    for (int m = 0; m < KB; ++m) {
      const int d0 = 16 * m + g;  // dims of rows g and g+8 of m-tile m
      if (hh0 < G) { s_o[warp][hh0][d0] = o[m][0]; s_o[warp][hh0][d0 + 8] = o[m][2]; }
      if (hh1 < G) { s_o[warp][hh1][d0] = o[m][1]; s_o[warp][hh1][d0 + 8] = o[m][3]; }
    }
  }
  __syncthreads();
  const int64_t out_base = ((int64_t)b * a.h_q + (int64_t)h * G) * D;
  float* part = nullptr;
  int* tickets = nullptr;
  if (splits > 1) {
    tickets = reinterpret_cast<int*>(a.ws);
    const int64_t n_pairs = (int64_t)gridDim.y;
    part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.ws) + ((n_pairs * 4 + 255) / 256) * 256);
  }
  for (int e = tid; e < G * D; e += kThreads) {
    const int row = e / D, dim = e % D;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, s_m[w][row]);
    float acc = 0.f, l = 0.f;
    if (mm != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = fast_exp2(s_m[w][row] - mm);
        acc += f * s_o[w][row][dim];
        l += f * s_l[w][row];
      }
    }
    if (splits == 1) {
      a.out[out_base + (int64_t)row * D + dim] = f_to_bf16(l > 0.f ? acc / l : 0.f);
    } else {
      float* pp = part + (((int64_t)pair * splits + split) * G + row) * (D + 2);
      __stcg(pp + 2 + dim, acc);
      if (dim == 0) {
        __stcg(pp, mm);
        __stcg(pp + 1, l);
      }
    }
  }
  if (splits == 1) return;

  // ---- last CTA of this (b, h) combines the partials -----------------------------------------
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&tickets[pair], 1) == splits - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const float* pbase = part + (int64_t)pair * splits * G * (D + 2);
  const int64_t step = (int64_t)G * (D + 2);  // floats per split
  if (splits * G * 3 * (int)sizeof(float) <= Ring<D>::kBytes) {
    // every split's (m, l) of every row into shared memory at once (the ring is free now), one
    // weight per (split, row) w = 2^(m - M) / L with M the rows' maximum and L the merged sum,
    // then each output element is one weighted sum of independent loads
    float* s_pm = reinterpret_cast<float*>(att_ring);
    float* s_pl = s_pm + splits * G;
    float* s_w = s_pl + splits * G;
    for (int i = tid; i < splits * G; i += kThreads) {
      const int sp = i / G, row = i % G;
      s_pm[i] = __ldcg(pbase + sp * step + (int64_t)row * (D + 2));
      s_pl[i] = __ldcg(pbase + sp * step + (int64_t)row * (D + 2) + 1);
    }
    __syncthreads();
    if (tid < G) {
      float mm = -INFINITY;
      for (int sp = 0; sp < splits; ++sp) mm = fmaxf(mm, s_pm[sp * G + tid]);
      float l = 0.f;
      if (mm != -INFINITY)
        for (int sp = 0; sp < splits; ++sp) l += fast_exp2(s_pm[sp * G + tid] - mm) * s_pl[sp * G + tid];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      for (int sp = 0; sp < splits; ++sp)
        s_w[sp * G + tid] = mm != -INFINITY ? fast_exp2(s_pm[sp * G + tid] - mm) * inv : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kThreads) {
      const int row = e / D, dim = e % D;
      const float* pp = pbase + (int64_t)row * (D + 2) + 2 + dim;
      float acc = 0.f;
#pragma unroll 8
      for (int sp = 0; sp < splits; ++sp) acc += s_w[sp * G + row] * __ldcg(pp + sp * step);
      a.out[out_base + (int64_t)row * D + dim] = f_to_bf16(acc);
    }
  } else {
    for (int e = tid; e < G * D; e += kThreads) {
      const int row = e / D, dim = e % D;
      const float* pp = pbase + (int64_t)row * (D + 2);
      float mm = -INFINITY;
      for (int s_ = 0; s_ < splits; ++s_) mm = fmaxf(mm, __ldcg(pp + s_ * step));
      float acc = 0.f, l = 0.f;
      if (mm != -INFINITY) {
        for (int s_ = 0; s_ < splits; ++s_) {
          const float f = fast_exp2(__ldcg(pp + s_ * step) - mm);
          acc += f * __ldcg(pp + s_ * step + 2 + dim);
          l += f * __ldcg(pp + s_ * step + 1);
        }
      }
      a.out[out_base + (int64_t)row * D + dim] = f_to_bf16(l > 0.f ? acc / l : 0.f);
    }
  }
  if (tid == 0) tickets[pair] = 0;
}

template <int D, bool INDEXED>
cudaError_t launch_t(const AttendArgs& a, const AttendPlan& plan, bool pdl, cudaStream_t s) {
  auto kern = attend_kernel<D, INDEXED>;
  constexpr int kRingBytes = Ring<D>::kBytes;
  static_assert(kRingBytes >= kWarps * kAttendMaxG * D * (int)sizeof(float), "merge buffer");
  cudaError_t ce = configure_kernel((const void*)kern, kRingBytes, false);
  if (ce != cudaSuccess) return ce;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.splits, a.batch * a.h_kv, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kRingBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, plan.chunk, plan.splits);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace attend_detail

AttendPlan plan_attend(int pairs, int positions, int group, int d) {
  AttendPlan p;
  const int unit = attend_detail::kWarps * attend_detail::kTile;  // 64 positions
  positions = positions < 1 ? 1 : positions;
  const int max_splits = (positions + unit - 1) / unit;
  // about one wave of resident CTAs (2 per SM at d = 128, 1 at d = 256); more splits only when
  // the pairs are few
  const int slots = (d == 128 ? 2 : 1) * num_sms();
  int splits = slots / (pairs > 0 ? pairs : 1);
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int chunk = (positions + splits - 1) / splits;
  chunk = (chunk + unit - 1) / unit * unit;
  if (chunk < 4 * unit) chunk = 4 * unit;  // at least 4 tiles per warp (fill the ring)
  if (chunk > attend_detail::kMaxChunk) chunk = attend_detail::kMaxChunk;
  splits = (positions + chunk - 1) / chunk;
  p.splits = splits;
  p.chunk = chunk;
  p.ws_bytes = splits > 1 ? (((size_t)pairs * 4 + 255) / 256) * 256 +
                                (size_t)pairs * splits * group * (d + 2) * sizeof(float)
                          : 0;
  return p;
}

cudaError_t launch_attend(const AttendArgs& a, bool indexed, const AttendPlan& plan, bool pdl,
                          cudaStream_t s) {
  if (a.batch * a.h_kv == 0) return cudaSuccess;
  if (a.d == 128)
    return indexed ? attend_detail::launch_t<128, true>(a, plan, pdl, s)
                   : attend_detail::launch_t<128, false>(a, plan, pdl, s);
  if (a.d == 256)
    return indexed ? attend_detail::launch_t<256, true>(a, plan, pdl, s)
                   : attend_detail::launch_t<256, false>(a, plan, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
