// Calibration, step 1: uncentred second moments of group-mean queries and keys per KV head
// (JSSA summary, Theoretical Foundation: the second-moment matrices of eq. (3), and section 3.2;
// JSSA README, section 2).
//
// G_K[h]    = sum_n k_n k_n^T
// G_Qbar[h] = sum_n qbar_n qbar_n^T = (1/G^2) sum_n sum_{g,g'} q_{n,g} q_{n,g'}^T
// Two forms of the query side:
//  * exact heads (G small): the second form keeps the tensor-core inputs exact: every q_{n,g} is
//    a bf16 value, so the G^2 products per sample are exact in the fp32 accumulators (qbar itself
//    is not bf16);
//  * mean planes (many heads per group, e.g. the 128 heads of a multi-head latent layer, where
//    G^2 products per sample would dominate): the CTA forms qbar in fp32 and splits it exactly
//    into three bf16 planes, qbar = hi + mid + lo (8 significant bits each), then sums the six
//    plane products hi.hi, hi.mid, mid.hi, hi.lo, lo.hi, mid.mid (the three it drops are below
//    2^-24 of the result).
//
// Grid (2 [keys | queries] x (d / 128)^2 tiles, h_kv, sample chunks); 8 warps per CTA tile one
// 128 x 128 block of the d x d Gram (warp w: rows 32*(w/2).., cols 64*(w%2).. of the block) with
// mma.sync m16n8k16. Sample tiles of 32 rows per head (or plane) are staged in swizzled shared
// memory; both operands are read with ldmatrix.trans (X^T X). Each CTA adds its chunk sum (fp32,
// folded per block) into the float64 totals. The blocks of one chunk are neighbours in the grid,
// so a chunk's query rows are read from HBM once and from L2 by the others.
#include "common.cuh"

namespace jssa {

namespace calib_detail {

constexpr int kThreads = 256;
constexpr int kTileN = 32;        // samples per staged tile
constexpr int kChunkN = 256;      // samples per CTA
constexpr int kPlanes = 3;        // bf16 planes of the group mean (mean-plane form)

// The group means of one tile's samples for the dimensions of two 128-dimension bands (the rows
// and the columns of this CTA's Gram block), split into kPlanes bf16 planes in the staged layout
// (plane p, sample r at row p * kTileN + r; 16-byte chunk c at c ^ (r & 7)).
template <int D>
__device__ __forceinline__ void stage_mean_planes(const uint16_t* __restrict__ q, int64_t q_stride,
                                                  int64_t q_hstride, int h, int G, int t0, int n,
                                                  int band_r, int band_c, uint32_t sbase) {
  constexpr int RB = D * 2;
  constexpr int kGroups = 128 / 8;  // 8-dimension groups per band
  const int n_bands = band_r == band_c ? 1 : 2;
  const float inv_g = 1.f / (float)G;
  for (int it = threadIdx.x; it < kTileN * kGroups * n_bands; it += kThreads) {
    const int r = it % kTileN;
    const int gi = (it / kTileN) % kGroups;
    const int band = it / (kTileN * kGroups);
    const int c8 = (band ? band_c : band_r) * kGroups + gi;  // 16-byte chunk of the row
    const int s = t0 + r;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    if (s < n) {
      const uint16_t* base = q + (int64_t)s * q_stride + (int64_t)h * G * q_hstride + c8 * 8;
      int g = 0;
      for (; g + 8 <= G; g += 8) {  // eight head rows in flight
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(g + u) * q_hstride));
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] += bf16_lo(w[e]);
            acc[2 * e + 1] += bf16_hi(w[e]);
          }
        }
      }
      for (; g < G; ++g) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)g * q_hstride));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += bf16_lo(w[e]);
          acc[2 * e + 1] += bf16_hi(w[e]);
        }
      }
    }
    uint32_t pl[kPlanes][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x0 = acc[2 * e] * inv_g, x1 = acc[2 * e + 1] * inv_g;
#pragma unroll
      for (int p = 0; p < kPlanes; ++p) {  // each plane rounds what the earlier planes left
        const uint32_t w = pack_bf16x2(x0, x1);
        pl[p][e] = w;
        x0 -= bf16_lo(w);
        x1 -= bf16_hi(w);
      }
    }
#pragma unroll
    for (int p = 0; p < kPlanes; ++p) {
      const int row = p * kTileN + r;
      const uint32_t dst = sbase + row * RB + ((c8 ^ (r & 7)) * 16);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pl[p][0]),
                   "r"(pl[p][1]), "r"(pl[p][2]), "r"(pl[p][3])
                   : "memory");
    }
  }
}

template <int D, bool MEAN>
__global__ void __launch_bounds__(kThreads)
    gram_kernel(const uint16_t* __restrict__ q, int64_t q_stride, int64_t q_hstride,
                const uint16_t* __restrict__ k, int64_t k_stride, int n, int h_q, int h_kv,
                double* __restrict__ gram_q, double* __restrict__ gram_k) {
  static_assert(D == 128 || D == 256 || D == 512, "one CTA tiles a 128 x 128 block of the Gram");
  constexpr int RB = D * 2;  // row bytes
  constexpr int T = D / 128;  // blocks per Gram row
  extern __shared__ __align__(128) uint8_t calib_smem[];
  const uint32_t sbase = smem_u32(calib_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const bool is_q = (blockIdx.x & 1) == 1;
  const int blk = blockIdx.x >> 1;  // Gram block (blk / T, blk % T)
  const int G = h_q / h_kv;
  // rows staged per sample: the G heads (exact form), the mean's planes, or the key
  const int nh = is_q ? (MEAN ? kPlanes : G) : 1;
  const int n0 = blockIdx.z * kChunkN, n1 = min(n, n0 + kChunkN);

  // Tensor-core fp32 accumulation is not round-to-nearest, so the mma accumulators only ever
  // hold the sum of one (head pair, 32-sample tile) block and are folded into a second set of
  // fp32 registers with ordinary rounded adds after each block.
  float acc[2][8][4], tot[2][8][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = tot[a][b][c] = 0.f;

  const int row0 = 128 * (blk / T) + 32 * (warp >> 1);  // first Gram row of this warp
  const int col0 = 128 * (blk % T) + 64 * (warp & 1);   // first Gram column

  for (int t0 = n0; t0 < n1; t0 += kTileN) {
    // stage [nh][kTileN][D] (row r of head gl at ((gl*kTileN + r) * RB), chunks swizzled by r)
    if (MEAN && is_q) {
      stage_mean_planes<D>(q, q_stride, q_hstride, h, G, t0, n, blk / T, blk % T, sbase);
    } else {
      const int total_chunks = nh * kTileN * (D / 8);
      for (int c = tid; c < total_chunks; c += kThreads) {
        const int ch = c % (D / 8);
        const int r = (c / (D / 8)) % kTileN;
        const int gl = c / ((D / 8) * kTileN);
        const int s = t0 + r;
        const uint16_t* src = is_q ? q + (int64_t)(s < n ? s : 0) * q_stride + (int64_t)(h * G + gl) * q_hstride
                                   : k + (int64_t)(s < n ? s : 0) * k_stride + (int64_t)h * D;
        const uint32_t dst = sbase + (gl * kTileN + r) * RB + ((ch ^ (r & 7)) * 16);
        cp_async16(dst, src + ch * 8, s < n ? 16 : 0);
      }
      cp_async_commit();
      cp_async_wait<0>();
    }
    __syncthreads();

    const int mat = lane >> 3;
#pragma unroll 1
    for (int ga = 0; ga < nh; ++ga) {
#pragma unroll 1
      for (int gb = 0; gb < nh; ++gb) {
        if (MEAN && is_q && ga + gb >= kPlanes) continue;  // products below 2^-24 of the result
#pragma unroll
        for (int ks = 0; ks < kTileN / 16; ++ks) {
          uint32_t af[2][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const int r = ks * 16 + (mat >> 1) * 8 + (lane & 7);
            const int c = (row0 + mt * 16) / 8 + (mat & 1);
            ldsm_x4_t(sbase + (ga * kTileN + r) * RB + ((c ^ (r & 7)) * 16), af[mt][0], af[mt][1],
                      af[mt][2], af[mt][3]);
          }
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            const int r = ks * 16 + (mat & 1) * 8 + (lane & 7);
            const int c = (col0 + np * 16) / 8 + (mat >> 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sbase + (gb * kTileN + r) * RB + ((c ^ (r & 7)) * 16), b0, b1, b2, b3);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              mma_bf16(acc[mt][2 * np], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b0, b1);
              mma_bf16(acc[mt][2 * np + 1], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b2, b3);
            }
          }
        }
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int b = 0; b < 8; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              tot[a][b][c] += acc[a][b][c];
              acc[a][b][c] = 0.f;
            }
      }
    }
    __syncthreads();
  }

  double* gram = (is_q ? gram_q : gram_k) + (int64_t)h * D * D;
  const double sc = (is_q && !MEAN) ? 1.0 / ((double)G * (double)G) : 1.0;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int i = row0 + mt * 16 + (lane >> 2);
      const int j = col0 + nt * 8 + 2 * (lane & 3);
      atomicAdd(&gram[(int64_t)i * D + j], sc * (double)tot[mt][nt][0]);
      atomicAdd(&gram[(int64_t)i * D + j + 1], sc * (double)tot[mt][nt][1]);
      atomicAdd(&gram[(int64_t)(i + 8) * D + j], sc * (double)tot[mt][nt][2]);
      atomicAdd(&gram[(int64_t)(i + 8) * D + j + 1], sc * (double)tot[mt][nt][3]);
    }
}

}  // namespace calib_detail

bool gram_mean_form(int h_q, int h_kv, int d) {
  const int G = h_q / h_kv;
  return G * d > 2048;  // the exact form stages G head rows per sample
}

cudaError_t launch_gram(const uint16_t* q, int64_t q_stride, int64_t q_hstride, const uint16_t* k,
                        int64_t k_stride, int n, int h_q, int h_kv, int d, double* gram_q,
                        double* gram_k, cudaStream_t s) {
  using namespace calib_detail;
  if (n <= 0 || h_kv <= 0) return cudaSuccess;
  const bool mean = gram_mean_form(h_q, h_kv, d);
  const int G = h_q / h_kv;
  const size_t smem = (size_t)(mean ? kPlanes : (G > 1 ? G : 1)) * kTileN * d * 2;
  void (*kern)(const uint16_t*, int64_t, int64_t, const uint16_t*, int64_t, int, int, int, double*,
               double*) = nullptr;
  if (d == 128) kern = mean ? gram_kernel<128, true> : gram_kernel<128, false>;
  else if (d == 256) kern = mean ? gram_kernel<256, true> : gram_kernel<256, false>;
  else if (d == 512) kern = mean ? gram_kernel<512, true> : gram_kernel<512, false>;
  else return cudaErrorInvalidValue;
  cudaError_t e = configure_kernel((const void*)kern, (int)smem, false);
  if (e != cudaSuccess) return e;
  const int blocks = (d / 128) * (d / 128);
  dim3 grid(2 * blocks, h_kv, (n + kChunkN - 1) / kChunkN);
  kern<<<grid, kThreads, smem, s>>>(q, q_stride, q_hstride, k, k_stride, n, h_q, h_kv, gram_q,
                                    gram_k);
  return cudaGetLastError();
}

}  // namespace jssa
