// Internal launch interface between the C ABI (api.cu) and the kernel translation units.
// Host-side argument checks happen in api.cu; the launchers below assume valid arguments.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace jssa {

constexpr int64_t kScoreMaxContext = 1 << 22;  // positions per sequence the score kernels plan for
constexpr int kAttendWarps = 4;
constexpr int kAttendTile = 16;            // tokens per warp-level tile
constexpr int kAttendMaxG = 8;             // query heads per KV head held in one m16 tile

struct ScorePlan {
  int chunk;       // positions per scan CTA (power of two, multiple of the page size)
  int n_chunks;    // scan CTAs per (sequence, KV head)
  size_t ws_bytes; // prep records + candidate counts + candidate keys/positions
};

// The new token of a decode step, stored by the score kernels' prep stage.
struct StoreNew {
  const uint16_t* k_new;  // bf16 [batch, h_kv, d]
  const uint16_t* v_new;  // bf16 [batch, h_kv, d], or null (a latent row is its own value)
  uint16_t* k_cache;
  uint16_t* v_cache;      // or null with v_new
  int64_t page_stride, slot_stride, head_stride;
  uint8_t* score_cache;
};

struct AttendPlan {
  int splits;      // CTAs per (sequence, KV head)
  int chunk;       // positions per CTA (multiple of 64)
  size_t ws_bytes; // tickets + partials
};

int num_sms();

// Raise a kernel's dynamic shared-memory limit (and allow clusters above 8 CTAs) once per device;
// later calls are lock-protected lookups, so launches stay cheap and safe under stream capture.
cudaError_t configure_kernel(const void* fn, int smem_bytes, bool nonportable_cluster);

ScorePlan plan_score(int pairs, int max_seq_len, int page_size, int d);
AttendPlan plan_attend(int pairs, int positions, int group, int d);

cudaError_t launch_store(const uint16_t* k, int64_t k_stride_t, const int64_t* slot_mapping,
                         int t, int h_kv, int d, int r, const float* basis, uint8_t* score_cache,
                         int64_t num_pages, int page_size, cudaStream_t s,
                         bool bf16_codes = false);

// Decode-time store: token b writes position seq_lens[b]-1 (K/V rows and scoring code).
cudaError_t launch_store_decode(const uint16_t* k_new, const uint16_t* v_new, uint16_t* k_cache,
                                uint16_t* v_cache, int64_t ps_stride, int64_t slot_stride,
                                int64_t head_stride, uint8_t* score_cache, const float* basis,
                                const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                                int batch, int h_kv, int d, int r, int64_t num_pages,
                                int page_size, cudaStream_t s);

cudaError_t launch_score_topk(const uint16_t* q, const float* basis, const uint8_t* score_cache,
                              const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                              int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                              int page_size, int budget, int32_t* idx, int32_t* count,
                              void* ws, int* attend_tickets, const StoreNew* store, bool pdl,
                              cudaStream_t s, bool bf16_codes = false, int tickets_per_pair = 1);

struct AttendArgs {
  const uint16_t* q;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  int64_t page_stride, slot_stride, head_stride;
  const int32_t* block_table;
  int max_pages;
  const int32_t* idx;       // indexed mode
  const int32_t* count;     // indexed mode
  const int32_t* seq_lens;  // dense mode
  int window;               // dense mode
  int batch, h_q, h_kv, d;
  int budget;               // indexed mode: index-set capacity
  int64_t num_pages;
  int page_size;
  float scale;
  uint16_t* out;
  void* ws;
};

cudaError_t launch_attend(const AttendArgs& a, bool indexed, const AttendPlan& plan, bool pdl,
                          cudaStream_t s);

cudaError_t launch_gather(const uint16_t* k_cache, const uint16_t* v_cache, int64_t page_stride,
                          int64_t slot_stride, int64_t head_stride, const int32_t* block_table,
                          int max_pages, const int32_t* idx, const int32_t* count, int batch,
                          int h_kv, int d, int budget, int64_t num_pages, int page_size,
                          uint16_t* k_out, uint16_t* v_out, int32_t* lens_out, cudaStream_t s);

// Multi-head latent attention over selected positions (absorbed form, 576-dim key rows,
// 512-dim values, 128 query heads x 128 value dimensions per CTA on the 5th-generation tensor
// cores): split-K plan and launch.
struct MlaPlan {
  int splits;  // 0: the budget is beyond what the split merge holds (unsupported)
  int chunk;
  size_t ws_bytes;
};
MlaPlan plan_mla(int batch, int h_q, int budget);
// Split counters of the latent attention per sequence (head blocks x value quarters).
int mla_tickets_per_sequence(int h_q);
// Clock-cycle limit of the tensor-core waits in a tile loop (default about one second).
long long tc_wait_limit();
void set_tc_wait_limit(long long cycles);  // <= 0: the default
cudaError_t launch_mla(const uint16_t* q, const uint16_t* kv, int64_t page_stride,
                       int64_t slot_stride, const int32_t* block_table, int max_pages,
                       const int32_t* idx, const int32_t* count, int batch, int h_q, int budget,
                       int64_t num_pages, int page_size, float scale, uint16_t* out, void* ws,
                       const MlaPlan& plan, bool pdl, cudaStream_t s, bool q_early = false);

// Second moments; q_hstride: elements between the head rows of one query sample.
cudaError_t launch_gram(const uint16_t* q, int64_t q_stride, int64_t q_hstride, const uint16_t* k,
                        int64_t k_stride, int n, int h_q, int h_kv, int d, double* gram_q,
                        double* gram_k, cudaStream_t s);

cudaError_t launch_basis(const double* gram_q, const double* gram_k, int h_kv, int d, int r,
                         float* basis, double* eigvals, double* ws, cudaStream_t s);

}  // namespace jssa
