// Gather-free indexed attention and the dense paged decode baseline (JSSA summary, section 3.1
// step 3 and section 3.3; JSSA README, section 3 microbenchmark against full-KV decode).
//
// Grid: (splits, batch * h_kv). A CTA owns one (sequence b, KV head h) and one contiguous range
// of its positions -- a slice of the index set (indexed mode) or of [lo, seq_len) (dense mode).
//   * Row addresses: the CTA first turns each of its positions into a 64-bit element offset
//     (page-table lookup, bounds checked) kept in shared memory.
//   * Each of the 4 warps walks its own 16-token tiles with a 3-stage cp.async pipeline: the K
//     and V rows (256 B each at d = 128) are copied straight from their paged locations into a
//     swizzled shared-memory tile -- no staging buffer in global memory.
//   * The G query heads of the KV head form the rows of an m16 tensor-core tile:
//     S = Q K^T and O += P V are mma.sync m16n8k16 (bf16 in, fp32 accumulate); P is split into a
//     bf16 high and low part so the probabilities keep ~16 significant bits.
//   * Online softmax in the log2 domain; warps merge in shared memory; CTAs of one (b, h) merge
//     through a float partial (m, l, o) in the workspace, the last CTA to take the ticket
//     combines them, writes the bf16 output and resets the ticket.
#include <float.h>

#include "common.cuh"

namespace jssa {

namespace attend_detail {

constexpr int kWarps = kAttendWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 3;
constexpr int kTile = kAttendTile;
constexpr int kMaxChunk = 1024;  // positions per CTA (row offsets kept in shared memory)

template <int D>
struct Smem {
  static constexpr int kRowBytes = D * 2;
  static constexpr int kTileBytes = kTile * kRowBytes;            // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;              // K + V
  static constexpr int kWarpBytes = kStages * kStageBytes;
  static constexpr int kPipeBytes = kWarps * kWarpBytes;
  static constexpr int kOffBytes = kMaxChunk * 8;
  static constexpr int kTotal = kPipeBytes + kOffBytes;
  // merge scratch (aliases the pipeline buffers after the main loop)
  static constexpr int kMergeBytes = kWarps * kAttendMaxG * (D + 2) * 4;
  static_assert(kMergeBytes <= kPipeBytes, "merge scratch");
};

template <int D, bool INDEXED>
__global__ void __launch_bounds__(kThreads, 2) attend_kernel(AttendArgs a, int chunk, int splits) {
  using S = Smem<D>;
  constexpr int CH = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t attend_smem[];
  int64_t* s_off = reinterpret_cast<int64_t*>(attend_smem + S::kPipeBytes);
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = blockIdx.y, split = blockIdx.x;
  const int b = pair / a.h_kv, h = pair % a.h_kv;
  const int G = a.h_q / a.h_kv;
  const int max_len = a.max_pages * a.page_size;

  // Q fragments (rows = the G query heads of this KV head; rows >= G are zero)
  uint32_t qa0[D / 16], qa2[D / 16];
  {
    const int row = lane >> 2;
    const uint32_t* qrow =
        reinterpret_cast<const uint32_t*>(a.q + ((int64_t)b * a.h_q + (int64_t)h * G + row) * D);
#pragma unroll
    for (int kb = 0; kb < D / 16; ++kb) {
      qa0[kb] = row < G ? qrow[kb * 8 + (lane & 3)] : 0u;
      qa2[kb] = row < G ? qrow[kb * 8 + 4 + (lane & 3)] : 0u;
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

  // ---- row offsets of this CTA's positions ---------------------------------------------------
  const int32_t* bt = a.block_table + (int64_t)b * a.max_pages;
  for (int j = tid; j < n_mine; j += kThreads) {
    int pos = INDEXED ? a.idx[(int64_t)pair * a.budget + j_begin + j] : lo + j_begin + j;
    int64_t off = -1;
    if (pos < 0 || pos >= max_len) {
      raise_flag(2u);
    } else {
      const int32_t pg = bt[pos / a.page_size];
      if (pg < 0 || (int64_t)pg >= a.num_pages) raise_flag(1u);
      else
        off = (int64_t)pg * a.page_stride + (int64_t)(pos % a.page_size) * a.slot_stride +
              (int64_t)h * a.head_stride;
    }
    s_off[j] = off;
  }
  __syncthreads();

  // ---- per-warp pipelined tiles --------------------------------------------------------------
  const int n_tiles = (n_mine + kTile - 1) / kTile;
  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;
  uint8_t* wbase = attend_smem + warp * S::kWarpBytes;
  const uint32_t wbase_s = smem_u32(wbase);

  auto issue = [&](int i) {
    if (i < my_tiles) {
      const int tile = warp + i * kWarps;
      const int r = lane & 15, half = lane >> 4;
      const int j = tile * kTile + r;
      const int64_t off = j < n_mine ? s_off[j] : -1;
      const uint32_t kdst = wbase_s + (i % kStages) * S::kStageBytes + r * S::kRowBytes;
      const uint32_t vdst = kdst + S::kTileBytes;
      const uint16_t* ksrc = off >= 0 ? a.k_cache + off : a.k_cache;
      const uint16_t* vsrc = off >= 0 ? a.v_cache + off : a.v_cache;
      const int nbytes = off >= 0 ? 16 : 0;
#pragma unroll
      for (int c = half; c < CH; c += 2) {
        const uint32_t sw = (uint32_t)((c ^ (r & 7)) * 16);
        cp_async16(kdst + sw, ksrc + c * 8, nbytes);
        cp_async16(vdst + sw, vsrc + c * 8, nbytes);
      }
    }
    cp_async_commit();
  };

  const float scale_log2 = a.scale * 1.4426950408889634f;
  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) issue(i);

  for (int i = 0; i < my_tiles; ++i) {
    issue(i + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const int tile = warp + i * kWarps;
    const uint32_t kbuf = wbase_s + (i % kStages) * S::kStageBytes;
    const uint32_t vbuf = kbuf + S::kTileBytes;

    // S = Q K^T for 16 tokens (two n8 tiles)
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int mat = lane >> 3;
      const int row = (mat >> 1) * 8 + (lane & 7);
#pragma unroll
      for (int kb = 0; kb < D / 16; ++kb) {
        const int c = 2 * kb + (mat & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbuf + row * S::kRowBytes + ((c ^ (row & 7)) * 16), b0, b1, b2, b3);
        mma_bf16(s0, qa0[kb], 0u, qa2[kb], 0u, b0, b1);
        mma_bf16(s1, qa0[kb], 0u, qa2[kb], 0u, b2, b3);
      }
    }
    // mask positions past the end or with an invalid row
    const int t0 = tile * kTile + 2 * (lane & 3);
    float x[4];
    {
      const int tt[4] = {t0, t0 + 1, t0 + 8, t0 + 9};
      const float sv[4] = {s0[0], s0[1], s1[0], s1[1]};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = tt[e] < n_mine && s_off[tt[e]] >= 0;
        x[e] = ok ? sv[e] * scale_log2 : -INFINITY;
      }
    }
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float corr = fast_exp2(m_run - m_use);
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = fast_exp2(x[e] - m_use);
    l_run = l_run * corr + (p[0] + p[1]) + (p[2] + p[3]);
    m_run = m_new;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= corr;
      o[n][1] *= corr;
    }
    // P (16 heads x 16 tokens) as an A operand, split into bf16 high + low parts
    const uint32_t ph0 = pack_bf16x2(p[0], p[1]);
    const uint32_t ph2 = pack_bf16x2(p[2], p[3]);
    const uint32_t pl0 = pack_bf16x2(p[0] - bf16_lo(ph0), p[1] - bf16_hi(ph0));
    const uint32_t pl2 = pack_bf16x2(p[2] - bf16_lo(ph2), p[3] - bf16_hi(ph2));
    {
      const int mat = lane >> 3;
      const int row = (mat & 1) * 8 + (lane & 7);
#pragma unroll
      for (int j = 0; j < D / 16; ++j) {
        const int c = 2 * j + (mat >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbuf + row * S::kRowBytes + ((c ^ (row & 7)) * 16), b0, b1, b2, b3);
        mma_bf16(o[2 * j], ph0, 0u, ph2, 0u, b0, b1);
        mma_bf16(o[2 * j], pl0, 0u, pl2, 0u, b0, b1);
        mma_bf16(o[2 * j + 1], ph0, 0u, ph2, 0u, b2, b3);
        mma_bf16(o[2 * j + 1], pl0, 0u, pl2, 0u, b2, b3);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();  // pipeline buffers are now reused as merge scratch

  // ---- merge the 4 warps ---------------------------------------------------------------------
  float* s_m = reinterpret_cast<float*>(attend_smem);          // [warps][8]
  float* s_l = s_m + kWarps * kAttendMaxG;              // [warps][8]
  float* s_o = s_l + kWarps * kAttendMaxG;              // [warps][8][D]
  {
    const int row = lane >> 2;
    if (row < G) {
      if ((lane & 3) == 0) {
        s_m[warp * kAttendMaxG + row] = m_run;
        s_l[warp * kAttendMaxG + row] = l_run;
      }
      float* dst = s_o + (warp * kAttendMaxG + row) * D + 2 * (lane & 3);
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        dst[8 * n] = o[n][0];
        dst[8 * n + 1] = o[n][1];
      }
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
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, s_m[w * kAttendMaxG + row]);
    float acc = 0.f, l = 0.f;
    if (mm != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = fast_exp2(s_m[w * kAttendMaxG + row] - mm);
        acc += f * s_o[(w * kAttendMaxG + row) * D + dim];
        l += f * s_l[w * kAttendMaxG + row];
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
  for (int e = tid; e < G * D; e += kThreads) {
    const int row = e / D, dim = e % D;
    const float* pp = part + ((int64_t)pair * splits * G + row) * (D + 2);
    const int64_t step = (int64_t)G * (D + 2);
    float mm = -INFINITY;
    for (int s = 0; s < splits; ++s) mm = fmaxf(mm, __ldcg(pp + s * step));
    float acc = 0.f, l = 0.f;
    if (mm != -INFINITY) {
      for (int s = 0; s < splits; ++s) {
        const float f = fast_exp2(__ldcg(pp + s * step) - mm);
        acc += f * __ldcg(pp + s * step + 2 + dim);
        l += f * __ldcg(pp + s * step + 1);
      }
    }
    a.out[out_base + (int64_t)row * D + dim] = f_to_bf16(l > 0.f ? acc / l : 0.f);
  }
  if (tid == 0) tickets[pair] = 0;
}

template <int D, bool INDEXED>
cudaError_t launch_t(const AttendArgs& a, const AttendPlan& plan, bool pdl, cudaStream_t s) {
  auto kern = attend_kernel<D, INDEXED>;
  const int smem = Smem<D>::kTotal;
  cudaError_t e = configure_kernel((const void*)kern, (int)smem, false);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.splits, a.batch * a.h_kv, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, kern, a, plan.chunk, plan.splits);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace attend_detail

AttendPlan plan_attend(int pairs, int positions, int group, int d) {
  AttendPlan p;
  const int unit = attend_detail::kWarps * attend_detail::kTile;  // 64 positions
  positions = positions < 1 ? 1 : positions;
  const int max_splits = (positions + unit - 1) / unit;
  const int want_ctas = 4 * num_sms();
  int splits = (want_ctas + pairs - 1) / pairs;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int chunk = (positions + splits - 1) / splits;
  chunk = (chunk + unit - 1) / unit * unit;
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
  if (a.d == 128) return indexed ? attend_detail::launch_t<128, true>(a, plan, pdl, s) : attend_detail::launch_t<128, false>(a, plan, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
