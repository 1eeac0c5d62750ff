// C ABI of libjssa.so (declared in include/jssa.h): host-side argument checks, workspace sizing
// and kernel chaining. Nothing here allocates device memory or synchronises (jssa_device_error
// excepted).
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "jssa.h"
#include "common.cuh"

namespace jssa {



namespace {
std::mutex g_cfg_mu;
std::map<std::pair<const void*, int>, int> g_cfg_smem;  // (kernel, device) -> configured bytes
int g_sms[64] = {0};
}  // namespace

namespace {
constexpr long long kDefaultWaitLimit = 2000000000ll;  // ~1 s at the boost clock
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};
}  // namespace

long long tc_wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }
void set_tc_wait_limit(long long cycles) {
  g_wait_limit.store(cycles > 0 ? cycles : kDefaultWaitLimit, std::memory_order_relaxed);
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

cudaError_t configure_kernel(const void* fn, int smem_bytes, bool nonportable_cluster) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_cfg_mu);
  const auto key = std::make_pair(fn, dev);
  auto it = g_cfg_smem.find(key);
  if (it != g_cfg_smem.end() && it->second >= smem_bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e == cudaSuccess && nonportable_cluster)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) g_cfg_smem[key] = smem_bytes;
  return e;
}

}  // namespace jssa

namespace {

using jssa::AttendArgs;

constexpr int kVersion = 100;  // 0.1.0
constexpr int64_t kMaxContext = jssa::kScoreMaxContext;
constexpr int kMlaMaxBudget = 256 * 1024;  // selected positions per sequence, latent attention
constexpr int kMaxCalibSamples = 256 * 65535;  // calibration samples per call (grid z of chunks)

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? JSSA_OK : (int)e; }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline cudaStream_t as_stream(jssa_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

bool supported_dr(int d, int r) {
  // d 576: a multi-head latent layer, r the rank of its latent basis (r + 64 code columns)
  return (d == 128 && (r == 16 || r == 32 || r == 64)) || (d == 256 && r == 64) || (d == 576 && r == 64);
}
bool supported_d(int d) { return d == 128 || d == 256; }

int check_heads(int h_q, int h_kv) {
  if (h_q <= 0 || h_kv <= 0 || h_q % h_kv) return JSSA_ERR_SHAPE;
  return JSSA_OK;
}

int check_paging(int max_pages, int64_t num_pages, int page_size) {
  if (max_pages <= 0 || num_pages <= 0 || page_size <= 0) return JSSA_ERR_SHAPE;
  if (page_size & (page_size - 1)) return JSSA_ERR_UNSUPPORTED;  // powers of two only
  if ((int64_t)max_pages * page_size > (int64_t)INT32_MAX / 2) return JSSA_ERR_SHAPE;
  return JSSA_OK;
}

int check_kv(const void* k_cache, const void* v_cache, int64_t page_stride, int64_t slot_stride,
             int64_t head_stride, int h_kv, int d, int page_size) {
  if (!k_cache || !v_cache) return JSSA_ERR_NULL;
  if (!aligned16(k_cache) || !aligned16(v_cache)) return JSSA_ERR_ALIGN;
  if (page_stride <= 0 || slot_stride <= 0 || head_stride <= 0) return JSSA_ERR_SHAPE;
  if ((page_stride | slot_stride | head_stride) & 7) return JSSA_ERR_ALIGN;  // 16-byte rows
  if (head_stride < d && slot_stride < d) return JSSA_ERR_SHAPE;
  (void)h_kv;
  (void)page_size;
  return JSSA_OK;
}

// eigenvectors [h_kv][d][d] float64; at d = 256 also the matrices [h_kv][d][d + 1] (they do not
// fit in shared memory)
size_t basis_ws_bytes(int h_kv, int d) {
  size_t n = (size_t)h_kv * d * d;
  if (d > 128) n += (size_t)h_kv * d * (d + 1);
  return n * sizeof(double);
}

size_t score_ws_bytes(int batch, int h_kv, int max_seq_len, int page_size, int d) {
  if (batch * h_kv == 0) return 0;
  return jssa::plan_score(batch * h_kv, max_seq_len, page_size, d).ws_bytes;
}

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

jssa::AttendPlan attend_plan_indexed(int batch, int h_q, int h_kv, int d, int budget) {
  return jssa::plan_attend(batch * h_kv, budget, h_q / h_kv, d);
}

jssa::AttendPlan attend_plan_dense(int batch, int h_q, int h_kv, int d, int max_seq_len) {
  return jssa::plan_attend(batch * h_kv, max_seq_len, h_q / h_kv, d);
}


size_t decode_ws_bytes(int batch, int h_q, int h_kv, int d, int max_seq_len, int page_size,
                       int budget) {
  return align256(attend_plan_indexed(batch, h_q, h_kv, d, budget).ws_bytes) +
         score_ws_bytes(batch, h_kv, max_seq_len, page_size, d);
}

// Device staging of one step of jssa_decode_host: q, k_new, v_new, out (each 256-byte aligned).
size_t host_set_bytes(int batch, int h_q, int h_kv, int d) {
  const size_t q = (size_t)batch * h_q * d * 2, kv = (size_t)batch * h_kv * d * 2;
  return 2 * align256(q) + 2 * align256(kv);
}

// Per-workspace state of jssa_decode_host: two copy streams, the events that order the two
// staging sets between them and the caller's stream, and which set the next call takes.
struct HostPipe {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t uploaded[2] = {}, decoded[2] = {}, downloaded[2] = {}, start = nullptr;
  cudaEvent_t mark_up = nullptr, mark_down = nullptr;
  bool used[2] = {false, false};
  bool fresh = true;  // the next call orders the copy streams after the caller's stream
  int next = 0;
};
std::mutex g_pipe_mu;
std::map<std::pair<int, const void*>, HostPipe> g_pipes;

cudaError_t host_pipe(const void* ws, bool create, HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  auto it = g_pipes.find({dev, ws});
  if (it != g_pipes.end()) {
    *out = &it->second;
    return cudaSuccess;
  }
  *out = nullptr;
  if (!create) return cudaSuccess;
  HostPipe p;
  if ((e = cudaStreamCreateWithFlags(&p.up, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaStreamCreateWithFlags(&p.down, cudaStreamNonBlocking)) != cudaSuccess) return e;
  cudaEvent_t* evs[] = {&p.uploaded[0], &p.uploaded[1], &p.decoded[0], &p.decoded[1],
                        &p.downloaded[0], &p.downloaded[1], &p.start, &p.mark_up, &p.mark_down};
  for (cudaEvent_t* ev : evs)
    if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
  *out = &(g_pipes[{dev, ws}] = p);
  return cudaSuccess;
}
}  // namespace

extern "C" {

const char* jssa_status_string(int status) {
  switch (status) {
    case JSSA_OK: return "ok";
    case JSSA_ERR_NULL: return "a required pointer is NULL";
    case JSSA_ERR_SHAPE: return "inconsistent or out-of-range sizes";
    case JSSA_ERR_UNSUPPORTED: return "no kernel instance for these sizes";
    case JSSA_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case JSSA_ERR_WORKSPACE: return "workspace missing or too small";
    case JSSA_ERR_DEVICE: return "no usable CUDA device";
    case JSSA_ERR_SCRATCH_LIMIT: return "sizes exceed the static scratch of the allocation-free entry point";
    default: break;
  }
  if (status > 0) return cudaGetErrorString((cudaError_t)status);
  return "unknown status";
}

int jssa_version(void) { return kVersion; }

long long jssa_set_wait_limit(long long cycles) {
  const long long prev = jssa::tc_wait_limit();
  jssa::set_tc_wait_limit(cycles);
  return prev;
}

int jssa_workspace_size(int fn, int batch, int h_q, int h_kv, int d, int max_pages,
                        int page_size, int budget, size_t* bytes) {
  if (!bytes) return JSSA_ERR_NULL;
  *bytes = 0;
  if (batch < 0 || d <= 0 || max_pages < 0 || page_size <= 0) return JSSA_ERR_SHAPE;
  if (page_size & (page_size - 1)) return JSSA_ERR_UNSUPPORTED;
  if ((int64_t)max_pages * page_size > (int64_t)INT32_MAX / 2) return JSSA_ERR_SHAPE;
  const int max_seq_len = max_pages * page_size;
  if (fn == JSSA_FN_COMPUTE_BASIS) {
    if (h_kv <= 0) return JSSA_ERR_SHAPE;
    *bytes = basis_ws_bytes(h_kv, d);
    return JSSA_OK;
  }
  int st = check_heads(h_q, h_kv);
  if (st) return st;
  switch (fn) {
    case JSSA_FN_SCORE_TOPK:
      *bytes = score_ws_bytes(batch, h_kv, max_seq_len, page_size, d);
      return JSSA_OK;
    case JSSA_FN_INDEXED_ATTEND:
      if (budget <= 0) return JSSA_ERR_SHAPE;
      *bytes = attend_plan_indexed(batch, h_q, h_kv, d, budget).ws_bytes;
      return JSSA_OK;
    case JSSA_FN_DECODE:
      if (budget <= 0) return JSSA_ERR_SHAPE;
      *bytes = decode_ws_bytes(batch, h_q, h_kv, d, max_seq_len, page_size, budget);
      return JSSA_OK;
    case JSSA_FN_DECODE_HOST:
      if (budget <= 0) return JSSA_ERR_SHAPE;
      *bytes = align256(decode_ws_bytes(batch, h_q, h_kv, d, max_seq_len, page_size, budget)) +
               2 * host_set_bytes(batch, h_q, h_kv, d);
      return JSSA_OK;
    case JSSA_FN_MLA_ATTEND:
    case JSSA_FN_MLA_DECODE:
      if (budget <= 0 || h_kv != 1 || d != 576 || h_q % 16) return JSSA_ERR_SHAPE;
      if (budget > kMlaMaxBudget || jssa::plan_mla(batch, h_q, budget).splits == 0)
        return JSSA_ERR_UNSUPPORTED;
      *bytes = jssa::plan_mla(batch, h_q, budget).ws_bytes;
      if (fn == JSSA_FN_MLA_DECODE)
        *bytes = align256(*bytes) + score_ws_bytes(batch, 1, max_seq_len, page_size, 576);
      return JSSA_OK;
    case JSSA_FN_DENSE_DECODE: {
      const int span = (budget > 0 && budget < max_seq_len) ? budget : max_seq_len;
      *bytes = attend_plan_dense(batch, h_q, h_kv, d, span).ws_bytes;
      return JSSA_OK;
    }
    default:
      return JSSA_ERR_SHAPE;
  }
}

int jssa_workspace_init(void* ws, size_t ws_bytes, jssa_stream_t stream) {
  if (ws_bytes == 0) return JSSA_OK;
  if (!ws) return JSSA_ERR_NULL;
  return cuda_status(cudaMemsetAsync(ws, 0, ws_bytes, as_stream(stream)));
}

static int calibrate_common(const jssa_bf16* q, int64_t q_stride_n, int64_t q_stride_head,
                            const jssa_bf16* k, int64_t k_stride_n, int n, int h_q, int h_kv,
                            int d, double* gram_q, double* gram_k, jssa_stream_t stream) {
  if (n < 0 || n > kMaxCalibSamples) return JSSA_ERR_SHAPE;
  int st = check_heads(h_q, h_kv);
  if (st) return st;
  if (!supported_d(d) && d != 512) return JSSA_ERR_UNSUPPORTED;
  if (n == 0) return JSSA_OK;
  if (!q || !k || !gram_q || !gram_k) return JSSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || (q_stride_n & 7) || (q_stride_head & 7) || (k_stride_n & 7))
    return JSSA_ERR_ALIGN;
  if (q_stride_head < d || q_stride_n < (int64_t)(h_q - 1) * q_stride_head + d ||
      k_stride_n < (int64_t)h_kv * d)
    return JSSA_ERR_SHAPE;
  return cuda_status(jssa::launch_gram(q, q_stride_n, q_stride_head, k, k_stride_n, n, h_q, h_kv,
                                       d, gram_q, gram_k, as_stream(stream)));
}

int jssa_calibrate_accumulate(const jssa_bf16* q, int64_t q_stride_n, const jssa_bf16* k,
                              int64_t k_stride_n, int n, int h_q, int h_kv, int d,
                              double* gram_q, double* gram_k, jssa_stream_t stream) {
  return calibrate_common(q, q_stride_n, d, k, k_stride_n, n, h_q, h_kv, d, gram_q, gram_k,
                          stream);
}

int jssa_mla_calibrate_accumulate(const jssa_bf16* q, int64_t q_stride_n, int64_t q_stride_head,
                                  const jssa_bf16* kv, int64_t kv_stride_n, int n, int h_q,
                                  double* gram_q, double* gram_k, jssa_stream_t stream) {
  // the latent part (first 512 dimensions) of each head's absorbed query and of each latent row
  return calibrate_common(q, q_stride_n, q_stride_head, kv, kv_stride_n, n, h_q, 1, 512, gram_q,
                          gram_k, stream);
}

int jssa_compute_basis(const double* gram_q, const double* gram_k, int h_kv, int d, int r,
                       float* basis, double* eigvals, void* ws, size_t ws_bytes,
                       jssa_stream_t stream) {
  if (h_kv <= 0 || r <= 0 || r > d) return JSSA_ERR_SHAPE;
  if (!supported_d(d) && d != 512) return JSSA_ERR_UNSUPPORTED;
  if (!gram_q || !gram_k || !basis) return JSSA_ERR_NULL;
  const size_t need = basis_ws_bytes(h_kv, d);
  if (!ws || ws_bytes < need) return JSSA_ERR_WORKSPACE;
  if (((uintptr_t)ws & 7u) != 0) return JSSA_ERR_ALIGN;
  return cuda_status(jssa::launch_basis(gram_q, gram_k, h_kv, d, r, basis, eigvals,
                                        static_cast<double*>(ws), as_stream(stream)));
}

static int store_codes(const jssa_bf16* k, int64_t k_stride_t, const int64_t* slot_mapping, int t,
                       int h_kv, int d, int r, const float* basis, void* score_cache,
                       int64_t num_pages, int page_size, jssa_stream_t stream, bool bf16) {
  if (t < 0 || h_kv <= 0 || num_pages <= 0 || page_size <= 0) return JSSA_ERR_SHAPE;
  if (page_size & (page_size - 1)) return JSSA_ERR_UNSUPPORTED;
  if (r <= 0 || r > d) return JSSA_ERR_SHAPE;
  if (bf16 ? !(d == 128 && r == 32) : !supported_dr(d, r)) return JSSA_ERR_UNSUPPORTED;
  if (t == 0) return JSSA_OK;
  if (!k || !slot_mapping || !basis || !score_cache) return JSSA_ERR_NULL;
  if (!aligned16(k) || (k_stride_t & 7) || !aligned16(score_cache) || !aligned16(basis))
    return JSSA_ERR_ALIGN;
  if (k_stride_t < (int64_t)h_kv * d) return JSSA_ERR_SHAPE;
  return cuda_status(jssa::launch_store(k, k_stride_t, slot_mapping, t, h_kv, d, r, basis,
                                        static_cast<uint8_t*>(score_cache), num_pages, page_size,
                                        as_stream(stream), bf16));
}

int jssa_store(const jssa_bf16* k, int64_t k_stride_t, const int64_t* slot_mapping, int t,
               int h_kv, int d, int r, const float* basis, uint8_t* score_cache,
               int64_t num_pages, int page_size, jssa_stream_t stream) {
  return store_codes(k, k_stride_t, slot_mapping, t, h_kv, d, r, basis, score_cache, num_pages,
                     page_size, stream, false);
}

int jssa_store_bf16(const jssa_bf16* k, int64_t k_stride_t, const int64_t* slot_mapping, int t,
                    int h_kv, int d, int r, const float* basis, jssa_bf16* score_cache,
                    int64_t num_pages, int page_size, jssa_stream_t stream) {
  return store_codes(k, k_stride_t, slot_mapping, t, h_kv, d, r, basis, score_cache, num_pages,
                     page_size, stream, true);
}

static int check_score_args(const jssa_bf16* q, const float* basis, const uint8_t* score_cache,
                            const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                            int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                            int page_size, int budget, const int32_t* idx, const int32_t* count) {
  if (batch < 0 || budget <= 0) return JSSA_ERR_SHAPE;
  int st = check_heads(h_q, h_kv);
  if (st) return st;
  if (r <= 0 || r > d) return JSSA_ERR_SHAPE;
  if (!supported_dr(d, r)) return JSSA_ERR_UNSUPPORTED;
  if ((st = check_paging(max_pages, num_pages, page_size))) return st;
  if ((int64_t)max_pages * page_size > kMaxContext) return JSSA_ERR_UNSUPPORTED;
  if ((int64_t)batch * h_kv > 65535) return JSSA_ERR_UNSUPPORTED;  // one grid row per pair
  if (batch == 0) return JSSA_OK;
  if (!q || !basis || !score_cache || !block_table || !seq_lens || !idx || !count)
    return JSSA_ERR_NULL;
  // (the prep reads each query row with 16-byte loads)
  if (!aligned16(score_cache) || !aligned16(basis) || !aligned16(q)) return JSSA_ERR_ALIGN;
  return JSSA_OK;
}

int jssa_score_topk(const jssa_bf16* q, const float* basis, const uint8_t* score_cache,
                    const int32_t* block_table, int max_pages, const int32_t* seq_lens, int batch,
                    int h_q, int h_kv, int d, int r, int64_t num_pages, int page_size, int budget,
                    int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                    jssa_stream_t stream) {
  int st = check_score_args(q, basis, score_cache, block_table, max_pages, seq_lens, batch, h_q,
                            h_kv, d, r, num_pages, page_size, budget, idx, count);
  if (st || batch == 0) return st;
  const size_t need = score_ws_bytes(batch, h_kv, max_pages * page_size, page_size, d);
  if (!ws || ws_bytes < need) return JSSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return JSSA_ERR_ALIGN;
  return cuda_status(jssa::launch_score_topk(q, basis, score_cache, block_table, max_pages,
                                             seq_lens, batch, h_q, h_kv, d, r, num_pages,
                                             page_size, budget, idx, count, ws, nullptr,
                                             nullptr, true, as_stream(stream)));
}

int jssa_score_topk_bf16(const jssa_bf16* q, const float* basis, const jssa_bf16* score_cache,
                         const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                         int batch, int h_q, int h_kv, int d, int r, int64_t num_pages,
                         int page_size, int budget, int32_t* idx, int32_t* count, void* ws,
                         size_t ws_bytes, jssa_stream_t stream) {
  const uint8_t* sc = reinterpret_cast<const uint8_t*>(score_cache);
  int st = check_score_args(q, basis, sc, block_table, max_pages, seq_lens, batch, h_q, h_kv, d,
                            r, num_pages, page_size, budget, idx, count);
  if (st || batch == 0) return st;
  if (!(d == 128 && r == 32)) return JSSA_ERR_UNSUPPORTED;
  const size_t need = score_ws_bytes(batch, h_kv, max_pages * page_size, page_size, d);
  if (!ws || ws_bytes < need) return JSSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return JSSA_ERR_ALIGN;
  return cuda_status(jssa::launch_score_topk(q, basis, sc, block_table, max_pages, seq_lens,
                                             batch, h_q, h_kv, d, r, num_pages, page_size, budget,
                                             idx, count, ws, nullptr, nullptr, true,
                                             as_stream(stream), true));
}

static int check_attend_common(const jssa_bf16* q, const jssa_bf16* k_cache,
                               const jssa_bf16* v_cache, int64_t ps, int64_t ss, int64_t hs,
                               const int32_t* block_table, int max_pages, int batch, int h_q,
                               int h_kv, int d, int64_t num_pages, int page_size,
                               const jssa_bf16* out) {
  if (batch < 0) return JSSA_ERR_SHAPE;
  int st = check_heads(h_q, h_kv);
  if (st) return st;
  if (!supported_d(d)) return JSSA_ERR_UNSUPPORTED;
  if (h_q / h_kv > jssa::kAttendMaxG) return JSSA_ERR_UNSUPPORTED;
  if ((st = check_paging(max_pages, num_pages, page_size))) return st;
  if (batch == 0) return JSSA_OK;
  if (!q || !block_table || !out) return JSSA_ERR_NULL;
  if ((st = check_kv(k_cache, v_cache, ps, ss, hs, h_kv, d, page_size))) return st;
  if (((uintptr_t)q & 3u) || ((uintptr_t)out & 1u)) return JSSA_ERR_ALIGN;
  return JSSA_OK;
}

int jssa_indexed_attend(const jssa_bf16* q, const jssa_bf16* k_cache, const jssa_bf16* v_cache,
                        int64_t kv_page_stride, int64_t kv_slot_stride, int64_t kv_head_stride,
                        const int32_t* block_table, int max_pages, const int32_t* idx,
                        const int32_t* count, int batch, int h_q, int h_kv, int d, int budget,
                        int64_t num_pages, int page_size, float softmax_scale, jssa_bf16* out,
                        void* ws, size_t ws_bytes, jssa_stream_t stream) {
  if (budget <= 0) return JSSA_ERR_SHAPE;
  int st = check_attend_common(q, k_cache, v_cache, kv_page_stride, kv_slot_stride,
                               kv_head_stride, block_table, max_pages, batch, h_q, h_kv, d,
                               num_pages, page_size, out);
  if (st || batch == 0) return st;
  if (!idx || !count) return JSSA_ERR_NULL;
  const jssa::AttendPlan plan = attend_plan_indexed(batch, h_q, h_kv, d, budget);
  if (plan.ws_bytes && (!ws || ws_bytes < plan.ws_bytes)) return JSSA_ERR_WORKSPACE;
  if (plan.ws_bytes && !aligned16(ws)) return JSSA_ERR_ALIGN;
  AttendArgs a = {};
  a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
  a.page_stride = kv_page_stride; a.slot_stride = kv_slot_stride; a.head_stride = kv_head_stride;
  a.block_table = block_table; a.max_pages = max_pages; a.idx = idx; a.count = count;
  a.batch = batch; a.h_q = h_q; a.h_kv = h_kv; a.d = d; a.budget = budget;
  a.num_pages = num_pages; a.page_size = page_size; a.scale = softmax_scale; a.out = out;
  a.ws = ws;
  return cuda_status(jssa::launch_attend(a, true, plan, false, as_stream(stream)));
}

int jssa_dense_decode(const jssa_bf16* q, const jssa_bf16* k_cache, const jssa_bf16* v_cache,
                      int64_t kv_page_stride, int64_t kv_slot_stride, int64_t kv_head_stride,
                      const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                      int batch, int h_q, int h_kv, int d, int64_t num_pages, int page_size,
                      int window, float softmax_scale, jssa_bf16* out, void* ws,
                      size_t ws_bytes, jssa_stream_t stream) {
  int st = check_attend_common(q, k_cache, v_cache, kv_page_stride, kv_slot_stride,
                               kv_head_stride, block_table, max_pages, batch, h_q, h_kv, d,
                               num_pages, page_size, out);
  if (st || batch == 0) return st;
  if (!seq_lens) return JSSA_ERR_NULL;
  int span = max_pages * page_size;
  if (window > 0 && window < span) span = window;
  const jssa::AttendPlan plan = jssa::plan_attend(batch * h_kv, span, h_q / h_kv, d);
  if (plan.ws_bytes && (!ws || ws_bytes < plan.ws_bytes)) return JSSA_ERR_WORKSPACE;
  if (plan.ws_bytes && !aligned16(ws)) return JSSA_ERR_ALIGN;
  AttendArgs a = {};
  a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
  a.page_stride = kv_page_stride; a.slot_stride = kv_slot_stride; a.head_stride = kv_head_stride;
  a.block_table = block_table; a.max_pages = max_pages; a.seq_lens = seq_lens;
  a.window = window; a.batch = batch; a.h_q = h_q; a.h_kv = h_kv; a.d = d; a.budget = 0;
  a.num_pages = num_pages; a.page_size = page_size; a.scale = softmax_scale; a.out = out;
  a.ws = ws;
  // programmatic dependent launch: the kernel waits for the preceding kernel before any read
  return cuda_status(jssa::launch_attend(a, false, plan, true, as_stream(stream)));
}

static int check_mla_kv(const jssa_bf16* q, const void* kv_cache, int64_t kv_page_stride,
                        int64_t kv_slot_stride, const jssa_bf16* out) {
  if (!q || !kv_cache || !out) return JSSA_ERR_NULL;
  if (kv_page_stride <= 0 || kv_slot_stride < 576) return JSSA_ERR_SHAPE;
  if (!aligned16(kv_cache) || !aligned16(q) || ((kv_page_stride | kv_slot_stride) & 7) ||
      !aligned16(out))
    return JSSA_ERR_ALIGN;
  return JSSA_OK;
}

int jssa_mla_decode(const jssa_bf16* q, const jssa_bf16* kv_new, jssa_bf16* kv_cache,
                    int64_t kv_page_stride, int64_t kv_slot_stride, uint8_t* score_cache,
                    const float* basis, const int32_t* block_table, int max_pages,
                    const int32_t* seq_lens, int batch, int h_q, int r, int64_t num_pages,
                    int page_size, int budget, float softmax_scale, int32_t* idx, int32_t* count,
                    jssa_bf16* out, void* ws, size_t ws_bytes, jssa_stream_t stream) {
  int st = check_score_args(q, basis, score_cache, block_table, max_pages, seq_lens, batch, h_q, 1,
                            576, r, num_pages, page_size, budget, idx, count);
  if (st || batch == 0) return st;
  if (h_q % 16 || budget > kMlaMaxBudget) return JSSA_ERR_UNSUPPORTED;
  if ((st = check_mla_kv(q, kv_cache, kv_page_stride, kv_slot_stride, out))) return st;
  if (kv_new && !aligned16(kv_new)) return JSSA_ERR_ALIGN;
  const jssa::MlaPlan plan = jssa::plan_mla(batch, h_q, budget);
  if (plan.splits == 0) return JSSA_ERR_UNSUPPORTED;
  // workspace: [latent attention tickets + partials | score candidates]; the select kernel clears
  // each sequence's tickets before the attention runs, so no prior clearing is needed
  const size_t score_ws = score_ws_bytes(batch, 1, max_pages * page_size, page_size, 576);
  const size_t attend_bytes = align256(plan.ws_bytes);
  if (!ws || ws_bytes < attend_bytes + score_ws) return JSSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return JSSA_ERR_ALIGN;
  void* attend_ws = ws;
  void* cand_ws = static_cast<uint8_t*>(ws) + attend_bytes;
  cudaStream_t s = as_stream(stream);
  jssa::StoreNew sn = {};
  if (kv_new) {
    sn.k_new = kv_new; sn.v_new = nullptr; sn.k_cache = kv_cache; sn.v_cache = nullptr;
    sn.page_stride = kv_page_stride; sn.slot_stride = kv_slot_stride; sn.head_stride = 0;
    sn.score_cache = score_cache;
  }
  cudaError_t e = jssa::launch_score_topk(
      q, basis, score_cache, block_table, max_pages, seq_lens, batch, h_q, 1, 576, r, num_pages,
      page_size, budget, idx, count, cand_ws,
      plan.ws_bytes ? static_cast<int*>(attend_ws) : nullptr, kv_new ? &sn : nullptr, true, s,
      false, jssa::mla_tickets_per_sequence(h_q));
  if (e != cudaSuccess) return (int)e;
  return cuda_status(jssa::launch_mla(q, kv_cache, kv_page_stride, kv_slot_stride, block_table,
                                      max_pages, idx, count, batch, h_q, budget, num_pages,
                                      page_size, softmax_scale, out,
                                      plan.ws_bytes ? attend_ws : nullptr, plan, true, s,
                                      /*q_early=*/true));
}

int jssa_mla_attend(const jssa_bf16* q, const jssa_bf16* kv_cache, int64_t kv_page_stride,
                    int64_t kv_slot_stride, const int32_t* block_table, int max_pages,
                    const int32_t* idx, const int32_t* count, int batch, int h_q, int budget,
                    int64_t num_pages, int page_size, float softmax_scale, jssa_bf16* out,
                    void* ws, size_t ws_bytes, jssa_stream_t stream) {
  if (batch < 0 || h_q <= 0 || budget <= 0) return JSSA_ERR_SHAPE;
  if (h_q % 16 || budget > kMlaMaxBudget) return JSSA_ERR_UNSUPPORTED;
  int st = check_paging(max_pages, num_pages, page_size);
  if (st) return st;
  if (batch == 0) return JSSA_OK;
  if (!q || !kv_cache || !block_table || !idx || !count || !out) return JSSA_ERR_NULL;
  if (kv_page_stride <= 0 || kv_slot_stride < 576) return JSSA_ERR_SHAPE;
  if (!aligned16(kv_cache) || !aligned16(q) || ((kv_page_stride | kv_slot_stride) & 7) ||
      !aligned16(out))
    return JSSA_ERR_ALIGN;
  const jssa::MlaPlan plan = jssa::plan_mla(batch, h_q, budget);
  if (plan.splits == 0) return JSSA_ERR_UNSUPPORTED;
  if (plan.ws_bytes && (!ws || ws_bytes < plan.ws_bytes)) return JSSA_ERR_WORKSPACE;
  if (plan.ws_bytes && !aligned16(ws)) return JSSA_ERR_ALIGN;
  return cuda_status(jssa::launch_mla(q, kv_cache, kv_page_stride, kv_slot_stride, block_table,
                                      max_pages, idx, count, batch, h_q, budget, num_pages,
                                      page_size, softmax_scale, out, ws, plan, true,
                                      as_stream(stream)));
}

int jssa_gather_kv(const jssa_bf16* k_cache, const jssa_bf16* v_cache, int64_t kv_page_stride,
                   int64_t kv_slot_stride, int64_t kv_head_stride, const int32_t* block_table,
                   int max_pages, const int32_t* idx, const int32_t* count, int batch, int h_kv,
                   int d, int budget, int64_t num_pages, int page_size, jssa_bf16* k_out,
                   jssa_bf16* v_out, int32_t* lens_out, jssa_stream_t stream) {
  if (batch < 0 || h_kv <= 0 || budget <= 0) return JSSA_ERR_SHAPE;
  if (!supported_d(d)) return JSSA_ERR_UNSUPPORTED;
  int st = check_paging(max_pages, num_pages, page_size);
  if (st) return st;
  if (batch == 0) return JSSA_OK;
  if (!block_table || !idx || !count || !k_out || !v_out || !lens_out) return JSSA_ERR_NULL;
  if ((st = check_kv(k_cache, v_cache, kv_page_stride, kv_slot_stride, kv_head_stride, h_kv, d,
                     page_size)))
    return st;
  if (!aligned16(k_out) || !aligned16(v_out)) return JSSA_ERR_ALIGN;
  return cuda_status(jssa::launch_gather(k_cache, v_cache, kv_page_stride, kv_slot_stride,
                                         kv_head_stride, block_table, max_pages, idx, count, batch,
                                         h_kv, d, budget, num_pages, page_size, k_out, v_out,
                                         lens_out, as_stream(stream)));
}

int jssa_decode(const jssa_bf16* q, const jssa_bf16* k_new, const jssa_bf16* v_new,
                jssa_bf16* k_cache, jssa_bf16* v_cache, int64_t kv_page_stride,
                int64_t kv_slot_stride, int64_t kv_head_stride, uint8_t* score_cache,
                const float* basis, const int32_t* block_table, int max_pages,
                const int32_t* seq_lens, int batch, int h_q, int h_kv, int d, int r,
                int64_t num_pages, int page_size, int budget, float softmax_scale,
                int32_t* idx, int32_t* count, jssa_bf16* out, void* ws, size_t ws_bytes,
                jssa_stream_t stream) {
  int st = check_score_args(q, basis, score_cache, block_table, max_pages, seq_lens, batch, h_q,
                            h_kv, d, r, num_pages, page_size, budget, idx, count);
  if (st) return st;
  st = check_attend_common(q, k_cache, v_cache, kv_page_stride, kv_slot_stride, kv_head_stride,
                           block_table, max_pages, batch, h_q, h_kv, d, num_pages, page_size, out);
  if (st || batch == 0) return st;
  if ((k_new == nullptr) != (v_new == nullptr)) return JSSA_ERR_NULL;
  if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return JSSA_ERR_ALIGN;
  const jssa::AttendPlan plan = attend_plan_indexed(batch, h_q, h_kv, d, budget);
  // workspace: [attention tickets + partials | score candidates]; the score kernel clears the
  // tickets of every (sequence, KV head) before the attention runs, so no prior clearing is needed
  const size_t score_ws = score_ws_bytes(batch, h_kv, max_pages * page_size, page_size, d);
  const size_t attend_bytes = align256(plan.ws_bytes);
  if (!ws || ws_bytes < attend_bytes + score_ws) return JSSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return JSSA_ERR_ALIGN;
  void* attend_ws = ws;
  void* cand_ws = static_cast<uint8_t*>(ws) + attend_bytes;
  cudaStream_t s = as_stream(stream);
  jssa::StoreNew sn = {};
  if (k_new) {
    sn.k_new = k_new; sn.v_new = v_new; sn.k_cache = k_cache; sn.v_cache = v_cache;
    sn.page_stride = kv_page_stride; sn.slot_stride = kv_slot_stride;
    sn.head_stride = kv_head_stride; sn.score_cache = score_cache;
  }
  cudaError_t e = jssa::launch_score_topk(q, basis, score_cache, block_table, max_pages, seq_lens,
                                          batch, h_q, h_kv, d, r, num_pages, page_size, budget,
                                          idx, count, cand_ws,
                                          plan.ws_bytes ? static_cast<int*>(attend_ws) : nullptr,
                                          k_new ? &sn : nullptr, true, s);
  if (e != cudaSuccess) return (int)e;
  AttendArgs a = {};
  a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
  a.page_stride = kv_page_stride; a.slot_stride = kv_slot_stride; a.head_stride = kv_head_stride;
  a.block_table = block_table; a.max_pages = max_pages; a.idx = idx; a.count = count;
  a.batch = batch; a.h_q = h_q; a.h_kv = h_kv; a.d = d; a.budget = budget;
  a.num_pages = num_pages; a.page_size = page_size; a.scale = softmax_scale; a.out = out;
  a.ws = plan.ws_bytes ? attend_ws : nullptr;
  return cuda_status(jssa::launch_attend(a, true, plan, true, s));
}

int jssa_decode_host(const jssa_bf16* q_host, const jssa_bf16* k_new_host,
                     const jssa_bf16* v_new_host, jssa_bf16* k_cache, jssa_bf16* v_cache,
                     int64_t kv_page_stride, int64_t kv_slot_stride, int64_t kv_head_stride,
                     uint8_t* score_cache, const float* basis, const int32_t* block_table,
                     int max_pages, const int32_t* seq_lens, int batch, int h_q, int h_kv, int d,
                     int r, int64_t num_pages, int page_size, int budget, float softmax_scale,
                     int32_t* idx, int32_t* count, jssa_bf16* out_host, void* ws,
                     size_t ws_bytes, jssa_stream_t stream) {
  if (!q_host || !out_host) return JSSA_ERR_NULL;
  if ((k_new_host == nullptr) != (v_new_host == nullptr)) return JSSA_ERR_NULL;
  if (batch < 0 || h_q <= 0 || h_kv <= 0 || d <= 0 || max_pages < 0 || page_size <= 0 ||
      budget <= 0)
    return JSSA_ERR_SHAPE;
  if (batch == 0) return JSSA_OK;
  const int max_seq_len = max_pages * page_size;
  const size_t dec = align256(decode_ws_bytes(batch, h_q, h_kv, d, max_seq_len, page_size, budget));
  const size_t set = host_set_bytes(batch, h_q, h_kv, d);
  if (!ws || ws_bytes < dec + 2 * set) return JSSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return JSSA_ERR_ALIGN;
  HostPipe* p = nullptr;
  cudaError_t e = host_pipe(ws, true, &p);
  if (e != cudaSuccess) return (int)e;
  cudaStream_t s = as_stream(stream);
  const size_t q_bytes = (size_t)batch * h_q * d * 2, kv_bytes = (size_t)batch * h_kv * d * 2;
  const int k = p->next;
  uint8_t* base = static_cast<uint8_t*>(ws) + dec + k * set;
  jssa_bf16* q_dev = reinterpret_cast<jssa_bf16*>(base);
  jssa_bf16* out_dev = reinterpret_cast<jssa_bf16*>(base + align256(q_bytes));
  jssa_bf16* kn_dev = reinterpret_cast<jssa_bf16*>(base + 2 * align256(q_bytes));
  jssa_bf16* vn_dev = reinterpret_cast<jssa_bf16*>(base + 2 * align256(q_bytes) + align256(kv_bytes));
  if (p->fresh) {  // copies after everything already enqueued on the caller's stream
    if ((e = cudaEventRecord(p->start, s)) != cudaSuccess) return (int)e;
    if ((e = cudaStreamWaitEvent(p->up, p->start, 0)) != cudaSuccess) return (int)e;
    if ((e = cudaStreamWaitEvent(p->down, p->start, 0)) != cudaSuccess) return (int)e;
    p->fresh = false;
  }
  // uploads: once the step two back has read this staging set
  if (p->used[k] && (e = cudaStreamWaitEvent(p->up, p->decoded[k], 0)) != cudaSuccess) return (int)e;
  if ((e = cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, p->up)) != cudaSuccess)
    return (int)e;
  if (k_new_host) {
    if ((e = cudaMemcpyAsync(kn_dev, k_new_host, kv_bytes, cudaMemcpyHostToDevice, p->up)) != cudaSuccess)
      return (int)e;
    if ((e = cudaMemcpyAsync(vn_dev, v_new_host, kv_bytes, cudaMemcpyHostToDevice, p->up)) != cudaSuccess)
      return (int)e;
  }
  if ((e = cudaEventRecord(p->uploaded[k], p->up)) != cudaSuccess) return (int)e;
  // the step: after its uploads and after the download of the step two back (same output buffer)
  if ((e = cudaStreamWaitEvent(s, p->uploaded[k], 0)) != cudaSuccess) return (int)e;
  if (p->used[k] && (e = cudaStreamWaitEvent(s, p->downloaded[k], 0)) != cudaSuccess) return (int)e;
  const int st = jssa_decode(q_dev, k_new_host ? kn_dev : nullptr, k_new_host ? vn_dev : nullptr,
                             k_cache, v_cache, kv_page_stride, kv_slot_stride, kv_head_stride,
                             score_cache, basis, block_table, max_pages, seq_lens, batch, h_q, h_kv,
                             d, r, num_pages, page_size, budget, softmax_scale, idx, count, out_dev,
                             ws, dec, stream);
  if (st != JSSA_OK) return st;
  if ((e = cudaEventRecord(p->decoded[k], s)) != cudaSuccess) return (int)e;
  // download, overlapping the next step
  if ((e = cudaStreamWaitEvent(p->down, p->decoded[k], 0)) != cudaSuccess) return (int)e;
  if ((e = cudaMemcpyAsync(out_host, out_dev, q_bytes, cudaMemcpyDeviceToHost, p->down)) != cudaSuccess)
    return (int)e;
  if ((e = cudaEventRecord(p->downloaded[k], p->down)) != cudaSuccess) return (int)e;
  p->used[k] = true;
  p->next = k ^ 1;
  return JSSA_OK;
}

int jssa_decode_host_join(const void* ws, jssa_stream_t stream) {
  if (!ws) return JSSA_ERR_NULL;
  HostPipe* p = nullptr;
  cudaError_t e = host_pipe(ws, false, &p);
  if (e != cudaSuccess) return (int)e;
  if (!p) return JSSA_OK;  // no step issued with this workspace
  cudaStream_t s = as_stream(stream);
  if ((e = cudaEventRecord(p->mark_up, p->up)) != cudaSuccess) return (int)e;
  if ((e = cudaEventRecord(p->mark_down, p->down)) != cudaSuccess) return (int)e;
  if ((e = cudaStreamWaitEvent(s, p->mark_up, 0)) != cudaSuccess) return (int)e;
  if ((e = cudaStreamWaitEvent(s, p->mark_down, 0)) != cudaSuccess) return (int)e;
  p->fresh = true;
  return JSSA_OK;
}

int jssa_device_error(uint32_t* flags, int clear, jssa_stream_t stream) {
  if (!flags) return JSSA_ERR_NULL;
  cudaStream_t s = as_stream(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return (int)e;
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, jssa::g_device_error, sizeof(v));
  if (e != cudaSuccess) return (int)e;
  *flags = v;
  if (clear) {
    const unsigned int zero = 0u;
    e = cudaMemcpyToSymbol(jssa::g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return (int)e;
  }
  return JSSA_OK;
}

}  // extern "C"
