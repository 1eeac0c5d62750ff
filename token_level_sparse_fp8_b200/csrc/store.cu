// Store step: FP8 E4M3 projected key c = e4m3(M_h k) for new tokens (JSSA summary, section 3.4
// "Projected Scoring Cache"; JSSA README, section 4 notes: r bytes per token and KV head).
//
// BF16 = true stores bf16(M_h k) instead (two bytes per dimension: the scoring-cache ablation).
//
// One CTA per (KV head, slice of code columns, range of tokens). The slice of the head's basis
// rows (all r rows up to r = 64; 32 rows for the 128 code columns of a latent row, where the
// whole basis would not fit) is staged in shared memory once, widened to float64; each warp takes
// one token at a time, lane j computes output j (and j+32, ...) of the slice as a float64 dot
// product over the projected dimensions and rounds it once. At decode the same kernel also writes
// the new token's K and V rows into the paged cache.
//
// Multi-head latent attention (d 576): the basis [r, 512] projects the 512 latent dimensions and
// the 64 rotary dimensions pass through as the last 64 code columns (JSSA README, section 4
// notes: the MLA basis is [1, r, kv_lora_rank]; JSSA summary, section 3.4: 64 latent + 64 RoPE
// scoring dimensions); their slices stage no basis and round the key's own values.
#include "common.cuh"

namespace jssa {

namespace store_detail {

constexpr int kStoreThreads = 256;
constexpr int kStoreWarps = kStoreThreads / 32;
constexpr int store_rows_per_cta(int r) { return r > 64 ? 32 : r; }

template <int D, int R, bool DECODE, bool BF16>
__global__ void __launch_bounds__(kStoreThreads)
    store_kernel(const uint16_t* __restrict__ k, int64_t k_stride_t,
                 const int64_t* __restrict__ slot_mapping, int t_count, int h_kv,
                 const float* __restrict__ basis, uint8_t* __restrict__ score_cache,
                 int64_t num_pages, int page_size, int tokens_per_block,
                 // decode-only arguments
                 const uint16_t* __restrict__ v_new, uint16_t* __restrict__ k_cache,
                 uint16_t* __restrict__ v_cache, int64_t page_stride, int64_t slot_stride,
                 int64_t head_stride, const int32_t* __restrict__ block_table, int max_pages,
                 const int32_t* __restrict__ seq_lens) {
  constexpr int RS = store_rows_per_cta(R);
  constexpr bool kLatent = D == 576;
  constexpr int PD = kLatent ? D - 64 : D;  // dimensions the basis projects
  constexpr int PR = kLatent ? R - 64 : R;  // basis rows (the projected code columns)
  static_assert(PR % RS == 0, "slices of projected columns");
  // both operands of the float64 products are widened once, when staged: the slice of basis
  // rows per CTA and each warp's key row per token
  extern __shared__ double store_smem[];
  double* s_m = store_smem;                        // [RS][PD+1]
  double* s_k = store_smem + RS * (PD + 1);        // [warps][D]
  const int h = blockIdx.x / (R / RS), r0 = (blockIdx.x % (R / RS)) * RS;
  const bool rope_slice = kLatent && r0 >= PR;     // code columns that copy rotary dimensions
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // the slice of basis rows, 16-byte loads (several in flight per thread) into the padded layout
  static_assert(PD % 4 == 0, "basis rows in 16-byte pieces");
  if (!rope_slice) {
    const float4* m_h = reinterpret_cast<const float4*>(basis + ((int64_t)h * PR + r0) * PD);
#pragma unroll 6
    for (int i = threadIdx.x; i < RS * PD / 4; i += kStoreThreads) {
      const float4 v = m_h[i];
      double* dst = s_m + (4 * i / PD) * (PD + 1) + (4 * i) % PD;
      dst[0] = v.x;
      dst[1] = v.y;
      dst[2] = v.z;
      dst[3] = v.w;
    }
  }
  __syncthreads();

  const int t0 = blockIdx.y * tokens_per_block;
  const int t1 = min(t_count, t0 + tokens_per_block);
  double* kw = s_k + warp * D;
  for (int t = t0 + warp; t < t1; t += kStoreWarps) {
    int64_t page, off;
    if (DECODE) {
      const int L = seq_lens[t];
      if (L <= 0 || L > max_pages * page_size) {
        if (L != 0 && lane == 0) raise_flag(4u);
        continue;
      }
      const int pos = L - 1;
      page = block_table[(int64_t)t * max_pages + pos / page_size];
      off = pos % page_size;
    } else {
      const int64_t slot = slot_mapping[t];
      if (slot < 0) continue;
      page = slot / page_size;
      off = slot % page_size;
    }
    if (page < 0 || page >= num_pages) {
      if (lane == 0) raise_flag(1u);
      continue;
    }
    const uint16_t* krow = k + (int64_t)t * k_stride_t + (int64_t)h * D;
    if (D != 128 && D != 256) {  // any even D: 32-bit words, lane-strided
      static_assert(D % 2 == 0, "head dim");
      const uint32_t* k32 = reinterpret_cast<const uint32_t*>(krow);
#pragma unroll
      for (int w = lane; w < D / 2; w += 32) {
        const uint32_t v = k32[w];
        kw[2 * w] = bf16_lo(v);
        kw[2 * w + 1] = bf16_hi(v);
      }
      if (DECODE) {
        const int64_t base = page * page_stride + off * slot_stride + (int64_t)h * head_stride;
        const uint32_t* v32 = reinterpret_cast<const uint32_t*>(v_new + (int64_t)t * k_stride_t + (int64_t)h * D);
#pragma unroll
        for (int w = lane; w < D / 2; w += 32) {
          reinterpret_cast<uint32_t*>(k_cache + base)[w] = k32[w];
          reinterpret_cast<uint32_t*>(v_cache + base)[w] = v32[w];
        }
      }
    }
    if (D == 128 || D == 256) {
      // D/32 consecutive elements per lane (8 bytes for D = 128)
      constexpr int E = D / 32;
      uint32_t kw32[E / 2];
      if (E == 4) {
        uint2 v = *reinterpret_cast<const uint2*>(krow + lane * 4);
        kw32[0] = v.x;
        kw32[1] = v.y;
      } else {
        uint4 v = *reinterpret_cast<const uint4*>(krow + lane * 8);
        kw32[0] = v.x; kw32[1] = v.y; kw32[2] = v.z; kw32[3] = v.w;
      }
#pragma unroll
      for (int e = 0; e < E / 2; ++e) {
        kw[lane * E + 2 * e] = bf16_lo(kw32[e]);
        kw[lane * E + 2 * e + 1] = bf16_hi(kw32[e]);
      }
      if (DECODE) {
        const int64_t base = page * page_stride + off * slot_stride + (int64_t)h * head_stride;
        const uint16_t* vrow = v_new + (int64_t)t * k_stride_t + (int64_t)h * D;
        if (E == 4) {
          *reinterpret_cast<uint2*>(k_cache + base + lane * 4) = make_uint2(kw32[0], kw32[1]);
          *reinterpret_cast<uint2*>(v_cache + base + lane * 4) =
              *reinterpret_cast<const uint2*>(vrow + lane * 4);
        } else {
          *reinterpret_cast<uint4*>(k_cache + base + lane * 8) =
              make_uint4(kw32[0], kw32[1], kw32[2], kw32[3]);
          *reinterpret_cast<uint4*>(v_cache + base + lane * 8) =
              *reinterpret_cast<const uint4*>(vrow + lane * 8);
        }
      }
    }
    __syncwarp();
    constexpr int RB = BF16 ? 2 * R : R;  // code bytes per token
    uint8_t* dst = score_cache + ((page * h_kv + h) * page_size + off) * RB + r0 * (RB / R);
#pragma unroll
    for (int j0 = 0; j0 < RS; j0 += 32) {
      const int j = j0 + lane;
      if (RS % 32 != 0 && j >= RS) continue;  // a slice narrower than the warp (r = 16)
      if (rope_slice) {  // a rotary dimension of the latent row, rounded once
        const double y = kw[PD + (r0 - PR) + j];
        if (BF16) reinterpret_cast<uint16_t*>(dst)[j] = f64_to_bf16(y);
        else dst[j] = f64_to_e4m3(y);
        continue;
      }
      const double* mrow = s_m + j * (PD + 1);
      // float64 dot product in four interleaved partial sums (short dependency chains), one
      // rounding at the end
      double acc0 = 0.0, acc1 = 0.0, acc2 = 0.0, acc3 = 0.0;
#pragma unroll 4
      for (int i = 0; i < PD; i += 4) {
        acc0 = fma(mrow[i], kw[i], acc0);
        acc1 = fma(mrow[i + 1], kw[i + 1], acc1);
        acc2 = fma(mrow[i + 2], kw[i + 2], acc2);
        acc3 = fma(mrow[i + 3], kw[i + 3], acc3);
      }
      const double acc = (acc0 + acc1) + (acc2 + acc3);
      if (BF16) reinterpret_cast<uint16_t*>(dst)[j] = f64_to_bf16(acc);
      else dst[j] = f64_to_e4m3(acc);
    }
    __syncwarp();
  }
  if (DECODE) pdl_trigger();
}

template <int D, int R, bool DECODE, bool BF16>
cudaError_t launch_store_t(dim3 grid, size_t smem, cudaStream_t s, const uint16_t* k,
                           int64_t k_stride_t, const int64_t* slot_mapping, int t, int h_kv,
                           const float* basis, uint8_t* score_cache, int64_t num_pages,
                           int page_size, int tpb, const uint16_t* v_new, uint16_t* k_cache,
                           uint16_t* v_cache, int64_t page_stride, int64_t slot_stride,
                           int64_t head_stride, const int32_t* block_table, int max_pages,
                           const int32_t* seq_lens) {
  auto kern = store_kernel<D, R, DECODE, BF16>;
  cudaError_t e = configure_kernel((const void*)kern, (int)smem, false);
  if (e != cudaSuccess) return e;
  kern<<<grid, kStoreThreads, smem, s>>>(k, k_stride_t, slot_mapping, t, h_kv, basis, score_cache,
                                         num_pages, page_size, tpb, v_new, k_cache, v_cache,
                                         page_stride, slot_stride, head_stride, block_table,
                                         max_pages, seq_lens);
  return cudaGetLastError();
}

template <bool DECODE, bool BF16 = false>
cudaError_t dispatch_store(int d, int r, int t, int h_kv, int tpb, cudaStream_t s,
                           const uint16_t* k, int64_t k_stride_t, const int64_t* slot_mapping,
                           const float* basis, uint8_t* score_cache, int64_t num_pages,
                           int page_size, const uint16_t* v_new, uint16_t* k_cache,
                           uint16_t* v_cache, int64_t page_stride, int64_t slot_stride,
                           int64_t head_stride, const int32_t* block_table, int max_pages,
                           const int32_t* seq_lens) {
  if (t <= 0) return cudaSuccess;
  // a latent layer (d 576, basis rank r over the 512 latent dimensions) has r + 64 code columns
  const int cols = d == 576 ? r + 64 : r;
  const int pd = d == 576 ? d - 64 : d;
  const int rs = store_rows_per_cta(cols);
  dim3 grid(h_kv * (cols / rs), (t + tpb - 1) / tpb);
  const size_t smem = (size_t)(rs * (pd + 1) + kStoreWarps * d) * sizeof(double);
#define JSSA_STORE_CASE(DD, RR)                                                                  \
  if (d == DD && cols == RR)                                                                     \
    return launch_store_t<DD, RR, DECODE, BF16>(grid, smem, s, k, k_stride_t, slot_mapping, t,   \
                                          h_kv,                                                  \
                                          basis, score_cache, num_pages, page_size, tpb, v_new,  \
                                          k_cache, v_cache, page_stride, slot_stride,            \
                                          head_stride, block_table, max_pages, seq_lens);
  if (BF16) {
    JSSA_STORE_CASE(128, 32)
    return cudaErrorInvalidValue;
  }
  JSSA_STORE_CASE(128, 16)
  JSSA_STORE_CASE(128, 32)
  JSSA_STORE_CASE(128, 64)
  JSSA_STORE_CASE(256, 64)
  if (!DECODE) {
    JSSA_STORE_CASE(576, 128)  // latent rows: rank-64 basis + 64 rotary columns
  }
#undef JSSA_STORE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace store_detail

cudaError_t launch_store(const uint16_t* k, int64_t k_stride_t, const int64_t* slot_mapping,
                         int t, int h_kv, int d, int r, const float* basis, uint8_t* score_cache,
                         int64_t num_pages, int page_size, cudaStream_t s, bool bf16_codes) {
  // tokens per CTA: many for bulk stores; for a few tokens (a decode step's) two per CTA, so
  // that more CTAs share the per-token products over the staged basis slices
  const int tpb = t >= 4096 ? 256 : (t >= 256 ? store_detail::kStoreWarps : 2);
  if (bf16_codes)
    return store_detail::dispatch_store<false, true>(d, r, t, h_kv, tpb, s, k, k_stride_t,
                               slot_mapping, basis, score_cache, num_pages, page_size, nullptr,
                               nullptr, nullptr, 0, 0, 0, nullptr, 0, nullptr);
  return store_detail::dispatch_store<false>(d, r, t, h_kv, tpb, s, k, k_stride_t, slot_mapping, basis,
                               score_cache, num_pages, page_size, nullptr, nullptr, nullptr, 0, 0,
                               0, nullptr, 0, nullptr);
}

cudaError_t launch_store_decode(const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_cache,
                                uint16_t* v_cache, int64_t page_stride, int64_t slot_stride,
                                int64_t head_stride, uint8_t* score_cache, const float* basis,
                                const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                                int batch, int h_kv, int d, int r, int64_t num_pages,
                                int page_size, cudaStream_t s) {
  return store_detail::dispatch_store<true>(d, r, batch, h_kv, store_detail::kStoreWarps, s, k_new, (int64_t)h_kv * d,
                              nullptr, basis, score_cache, num_pages, page_size, v_new, k_cache,
                              v_cache, page_stride, slot_stride, head_stride, block_table,
                              max_pages, seq_lens);
}

}  // namespace jssa
