// Calibration, step 1: uncentred second moments of group-mean queries and keys per KV head
// (JSSA summary, Theoretical Foundation: the second-moment matrices of eq. (3), and section 3.2;
// JSSA README, section 2).
//
// G_K[h]    = sum_n k_n k_n^T
// G_Qbar[h] = sum_n qbar_n qbar_n^T = (1/G^2) sum_n sum_{g,g'} q_{n,g} q_{n,g'}^T
// The second form keeps the tensor-core inputs exact: every q_{n,g} is a bf16 value, so the
// G^2 products per sample are exact in the fp32 accumulators (qbar itself is not bf16).
//
// Grid (sample chunks, h_kv, 2 [keys | queries] x (d / 128)^2 tiles); 8 warps per CTA tile one
// 128 x 128 block of the d x d Gram (warp w: rows 32*(w/2).., cols 64*(w%2).. of the block) with
// mma.sync m16n8k16. Sample tiles of 32 rows
// per head are staged in swizzled shared memory with cp.async; both operands are read with
// ldmatrix.trans (X^T X). Each CTA adds its chunk sum (fp32, folded per block) into the float64
// totals.
#include "common.cuh"

namespace jssa {

namespace calib_detail {

constexpr int kThreads = 256;
constexpr int kTileN = 32;        // samples per staged tile
constexpr int kChunkN = 256;      // samples per CTA

template <int D>
__global__ void __launch_bounds__(kThreads)
    gram_kernel(const uint16_t* __restrict__ q, int64_t q_stride, const uint16_t* __restrict__ k,
                int64_t k_stride, int n, int h_q, int h_kv, double* __restrict__ gram_q,
                double* __restrict__ gram_k) {
  static_assert(D == 128 || D == 256, "one CTA tiles a 128 x 128 block of the Gram");
  constexpr int RB = D * 2;  // row bytes
  constexpr int T = D / 128;  // blocks per Gram row
  extern __shared__ __align__(128) uint8_t calib_smem[];
  const uint32_t sbase = smem_u32(calib_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.y;
  const bool is_q = (blockIdx.z & 1) == 1;
  const int blk = blockIdx.z >> 1;  // Gram block (blk / T, blk % T)
  const int G = h_q / h_kv;
  const int nh = is_q ? G : 1;  // head rows staged per sample
  const int n0 = blockIdx.x * kChunkN, n1 = min(n, n0 + kChunkN);

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
    const int total_chunks = nh * kTileN * (D / 8);
    for (int c = tid; c < total_chunks; c += kThreads) {
      const int ch = c % (D / 8);
      const int r = (c / (D / 8)) % kTileN;
      const int gl = c / ((D / 8) * kTileN);
      const int s = t0 + r;
      const uint16_t* src = is_q ? q + (int64_t)(s < n ? s : 0) * q_stride + (int64_t)(h * G + gl) * D
                                 : k + (int64_t)(s < n ? s : 0) * k_stride + (int64_t)h * D;
      const uint32_t dst = sbase + (gl * kTileN + r) * RB + ((ch ^ (r & 7)) * 16);
      cp_async16(dst, src + ch * 8, s < n ? 16 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int mat = lane >> 3;
#pragma unroll 1
    for (int ga = 0; ga < nh; ++ga) {
#pragma unroll 1
      for (int gb = 0; gb < nh; ++gb) {
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
  const double sc = is_q ? 1.0 / ((double)G * (double)G) : 1.0;
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

cudaError_t launch_gram(const uint16_t* q, int64_t q_stride, const uint16_t* k, int64_t k_stride,
                        int n, int h_q, int h_kv, int d, double* gram_q, double* gram_k,
                        cudaStream_t s) {
  if (n <= 0 || h_kv <= 0) return cudaSuccess;
  if (d != 128 && d != 256) return cudaErrorInvalidValue;
  const int G = h_q / h_kv;
  const size_t smem = (size_t)G * calib_detail::kTileN * d * 2;
  auto kern = d == 128 ? calib_detail::gram_kernel<128> : calib_detail::gram_kernel<256>;
  cudaError_t e = configure_kernel((const void*)kern, (int)smem, false);
  if (e != cudaSuccess) return e;
  const int blocks = (d / 128) * (d / 128);
  dim3 grid((n + calib_detail::kChunkN - 1) / calib_detail::kChunkN, h_kv, 2 * blocks);
  kern<<<grid, calib_detail::kThreads, smem, s>>>(q, q_stride, k, k_stride, n, h_q, h_kv, gram_q, gram_k);
  return cudaGetLastError();
}

}  // namespace jssa
