// Gather-free indexed attention and the dense paged decode baseline (JSSA summary, section 3.1
// step 3 and section 3.3; JSSA README, section 3 microbenchmark against full-KV decode).
//
// Grid: (splits, batch * h_kv). A CTA owns one (sequence b, KV head h) and one contiguous range
// of its positions -- a slice of the index set (indexed mode) or of [lo, seq_len) (dense mode).
//   * Row addresses: the CTA first turns each of its positions into a 64-bit element offset
//     (page-table lookup, bounds checked) kept in shared memory.
//   * Each of the 4 warps walks its own 16-token tiles. A tile's K and V rows (256 B each at
//     d = 128) are loaded with 16-byte non-allocating loads straight from their paged locations
//     into registers -- no staging buffer in global or shared memory -- and the next tile's loads
//     are in flight while the current tile is computed.
//   * Tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate) with the 16 tokens as the M
//     rows and the G <= 8 query heads of the KV head as the N columns: S^T = K Q^T, then
//     O^T += V^T P^T. The head dimension is visited in a fixed permuted order (the same for q and
//     k, and undone when O is written) so that every lane's fragment elements are contiguous in
//     the row: a lane reads 64 B of each of its two K rows and 32 B of each of its four V rows.
//     P^T reaches the B-operand layout with movmatrix, split into a bf16 high and low part so the
//     probabilities keep ~16 significant bits.
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

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

template <int D>
struct TileRegs {
  uint4 k[2][D / 32];   // rows g, g+8 of the tile: bytes [t * D/2, +D/2)
  uint4 v[4][D / 64];   // rows 2t, 2t+1, 8+2t, 9+2t: bytes [g * D/4, +D/4)
};

template <int D>
__device__ __forceinline__ void load_tile(TileRegs<D>& tr, const uint16_t* __restrict__ kc,
                                          const uint16_t* __restrict__ vc, const int64_t* s_off,
                                          int tile, int n_mine, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int j0 = tile * kTile;
  const int krow[2] = {g, g + 8};
  const int vrow[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int j = j0 + krow[i];
    const int64_t off = j < n_mine ? s_off[j] : -1;
    const uint16_t* src = kc + (off >= 0 ? off : 0) + t * (D / 4);
#pragma unroll
    for (int c = 0; c < D / 32; ++c)
      tr.k[i][c] = off >= 0 ? ld_stream_v4(src + c * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = j0 + vrow[i];
    const int64_t off = j < n_mine ? s_off[j] : -1;
    const uint16_t* src = vc + (off >= 0 ? off : 0) + g * (D / 8);
#pragma unroll
    for (int c = 0; c < D / 64; ++c)
      tr.v[i][c] = off >= 0 ? ld_stream_v4(src + c * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
}

__device__ __forceinline__ uint32_t word(const uint4& u, int i) {
  return i == 0 ? u.x : (i == 1 ? u.y : (i == 2 ? u.z : u.w));
}

template <int D, bool INDEXED>
__global__ void __launch_bounds__(kThreads, 2) attend_kernel(AttendArgs a, int chunk, int splits) {
  static_assert(D == 128, "head dim");
  constexpr int KB = D / 16;  // k-blocks of S^T, m-tiles of O^T
  __shared__ int64_t s_off[kMaxChunk];
  __shared__ float s_m[kWarps][kAttendMaxG], s_l[kWarps][kAttendMaxG];
  __shared__ float s_o[kWarps][kAttendMaxG][D];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int pair = blockIdx.y, split = blockIdx.x;
  const int b = pair / a.h_kv, h = pair % a.h_kv;
  const int G = a.h_q / a.h_kv;
  const int max_len = a.max_pages * a.page_size;

  // Q^T fragments (B operand of S^T = K Q^T): column n = head g of this KV head (zero for g >= G);
  // k-slot 16kb+2t+e <-> physical dim D/4*t + 4kb + e, 16kb+8+2t+e <-> D/4*t + 4kb + 2 + e
  uint32_t qb0[KB], qb1[KB];
  {
    const uint4* qrow = reinterpret_cast<const uint4*>(
        a.q + ((int64_t)b * a.h_q + (int64_t)h * G + (g < G ? g : 0)) * D + t * (D / 4));
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      const uint4 v = g < G ? qrow[c] : make_uint4(0u, 0u, 0u, 0u);
      qb0[2 * c] = v.x;
      qb1[2 * c] = v.y;
      qb0[2 * c + 1] = v.z;
      qb1[2 * c + 1] = v.w;
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
    const int pos = INDEXED ? a.idx[(int64_t)pair * a.budget + j_begin + j] : lo + j_begin + j;
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

  // ---- per-warp tiles, next tile's loads in flight ------------------------------------------
  const int n_tiles = (n_mine + kTile - 1) / kTile;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  float o[KB][4];
#pragma unroll
  for (int m = 0; m < KB; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};  // heads 2t, 2t+1

  TileRegs<D> cur, nxt;
  int tile = warp;
  if (tile < n_tiles) load_tile<D>(cur, a.k_cache, a.v_cache, s_off, tile, n_mine, lane);
  for (; tile < n_tiles; tile += kWarps) {
    if (tile + kWarps < n_tiles)
      load_tile<D>(nxt, a.k_cache, a.v_cache, s_off, tile + kWarps, n_mine, lane);

    // S^T (16 tokens x 8 heads) = K Q^T
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
      const int c = kb >> 1, w0 = (kb & 1) * 2;
      const uint32_t a0 = word(cur.k[0][c], w0), a2 = word(cur.k[0][c], w0 + 1);
      const uint32_t a1 = word(cur.k[1][c], w0), a3 = word(cur.k[1][c], w0 + 1);
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
    // O^T (dims x heads) += V^T P^T; m-tile m: rows g, g+8 = physical dims D/8*g + 2m, +1
#pragma unroll
    for (int m = 0; m < KB; ++m) {
      const int c = m >> 2, wi = m & 3;
      const uint32_t r0 = word(cur.v[0][c], wi), r1 = word(cur.v[1][c], wi);
      const uint32_t r2 = word(cur.v[2][c], wi), r3 = word(cur.v[3][c], wi);
      const uint32_t va0 = prmt(r0, r1, 0x5410u), va1 = prmt(r0, r1, 0x7632u);
      const uint32_t va2 = prmt(r2, r3, 0x5410u), va3 = prmt(r2, r3, 0x7632u);
      mma_bf16(o[m], va0, va1, va2, va3, bh0, bh1);
      mma_bf16(o[m], va0, va1, va2, va3, bl0, bl1);
    }
    cur = nxt;
  }
#pragma unroll
  for (int sh = 4; sh < 32; sh <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], sh);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], sh);
  }

  // ---- merge the 4 warps ---------------------------------------------------------------------
  {
    const int hh0 = 2 * t, hh1 = 2 * t + 1;
    if (g == 0) {
      if (hh0 < G) { s_m[warp][hh0] = m_run[0]; s_l[warp][hh0] = l_run[0]; }
      if (hh1 < G) { s_m[warp][hh1] = m_run[1]; s_l[warp][hh1] = l_run[1]; }
    }
#pragma unroll
    for (int m = 0; m < KB; ++m) {
      const int d0 = (D / 8) * g + 2 * m;  // physical dims of rows g and g+8 of m-tile m
      if (hh0 < G) { s_o[warp][hh0][d0] = o[m][0]; s_o[warp][hh0][d0 + 1] = o[m][2]; }
      if (hh1 < G) { s_o[warp][hh1][d0] = o[m][1]; s_o[warp][hh1][d0 + 1] = o[m][3]; }
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
  for (int e = tid; e < G * D; e += kThreads) {
    const int row = e / D, dim = e % D;
    const float* pp = part + ((int64_t)pair * splits * G + row) * (D + 2);
    const int64_t step = (int64_t)G * (D + 2);
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
  if (tid == 0) tickets[pair] = 0;
}

template <int D, bool INDEXED>
cudaError_t launch_t(const AttendArgs& a, const AttendPlan& plan, bool pdl, cudaStream_t s) {
  auto kern = attend_kernel<D, INDEXED>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.splits, a.batch * a.h_kv, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
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
  // about one wave of resident CTAs (2 per SM); more splits only when the pairs are few
  const int slots = 2 * num_sms();
  int splits = slots / (pairs > 0 ? pairs : 1);
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
  if (a.d == 128)
    return indexed ? attend_detail::launch_t<128, true>(a, plan, pdl, s)
                   : attend_detail::launch_t<128, false>(a, plan, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace jssa
