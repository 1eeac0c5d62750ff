// Allocation-free variant of the gather-free indexed attention (jssa_indexed_attend_noalloc).
//
// Some callers cannot hand the library a workspace: code that runs where device allocation is
// not allowed or not wanted (an inference runtime that owns every byte of device memory through
// its own pool and gives plug-ins no allocator, a latency-critical loop where cudaMalloc's
// implicit device synchronisation is unacceptable, or a host process that only links the C ABI
// and has no allocator of its own). For them this entry point keeps the split-K scratch (the
// per-(sequence, KV head) ticket counters and the fp32 partial results) in a file-scope device
// array of fixed size instead of a caller-provided workspace.
//
// The array lives in every GPU that loads the library until the process exits. In host code its
// name only stands for the symbol; the device address is looked up with cudaGetSymbolAddress
// (on the first call made with that device current, and again after the device's context was
// reset) and cached. Calls share
// the array: it keeps the previous call's contents, the ticket counters are cleared on the
// stream before every launch, and calls that overlap on the GPU (other streams, other threads)
// race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "jssa.h"
#include "common.cuh"

namespace jssa {
namespace noalloc_detail {

static __device__ __align__(256) unsigned char g_attend_scratch[JSSA_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;

// The cached address of g_attend_scratch per device, with the unique id of the CUDA context it
// was looked up in: cudaDeviceReset (or any teardown of the device's primary context) makes a
// new context, whose module copy of the array may sit elsewhere, so a changed id repeats the
// lookup.
struct ScratchSlot {
  void* addr;
  unsigned long long ctx_id;
};
ScratchSlot g_slot[64] = {};

// Driver entry points for the current context and its process-unique id, fetched once through
// the runtime (no link against the driver library is needed).
typedef int (*CtxGetCurrentFn)(void** ctx);
typedef int (*CtxGetIdFn)(void* ctx, unsigned long long* id);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
std::once_flag g_entry_once;

// Unique id of the calling thread's current context, or 0 when there is none yet or the driver
// does not provide the query.
unsigned long long current_context_id() {
  std::call_once(g_entry_once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  if (!g_ctx_current || !g_ctx_id) return 0ull;
  void* ctx = nullptr;
  unsigned long long id = 0ull;
  if (g_ctx_current(&ctx) != 0 || ctx == nullptr) return 0ull;
  if (g_ctx_id(ctx, &id) != 0) return 0ull;
  return id;
}

// Device address of g_attend_scratch on the current device. The set-up (cudaGetSymbolAddress
// with the device current) runs on the first call for a device and again whenever the device's
// context changed since; other calls return the cached address. Without a context id from the
// driver the lookup runs on every call.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long id = current_context_id();
  if (id != 0ull && g_slot[dev].addr != nullptr && g_slot[dev].ctx_id == id) {
    *out = g_slot[dev].addr;
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_attend_scratch);
  if (e != cudaSuccess) return e;
  g_slot[dev].addr = p;
  g_slot[dev].ctx_id = current_context_id();  // the lookup made the context current if needed
  *out = p;
  return cudaSuccess;
}

}  // namespace noalloc_detail
}  // namespace jssa

extern "C" int jssa_indexed_attend_noalloc(const jssa_bf16* q, const jssa_bf16* k_cache,
                                           const jssa_bf16* v_cache, int64_t kv_page_stride,
                                           int64_t kv_slot_stride, int64_t kv_head_stride,
                                           const int32_t* block_table, int max_pages,
                                           const int32_t* idx, const int32_t* count, int batch,
                                           int h_q, int h_kv, int d, int budget,
                                           int64_t num_pages, int page_size, float softmax_scale,
                                           jssa_bf16* out, jssa_stream_t stream) {
  if (budget <= 0) return JSSA_ERR_SHAPE;
  int st = check_attend_common(q, k_cache, v_cache, kv_page_stride, kv_slot_stride,
                               kv_head_stride, block_table, max_pages, batch, h_q, h_kv, d,
                               num_pages, page_size, out);
  if (st || batch == 0) return st;
  if (!idx || !count) return JSSA_ERR_NULL;
  const jssa::AttendPlan plan = attend_plan_indexed(batch, h_q, h_kv, d, budget);
  if (plan.ws_bytes > (size_t)JSSA_NOALLOC_SCRATCH_BYTES) return JSSA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  cudaError_t e = jssa::noalloc_detail::scratch_address(&scratch);
  if (e != cudaSuccess) return (int)e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (plan.ws_bytes) {
    // ticket counters must start at zero; the partials are written before they are read
    const size_t ticket_bytes = (((size_t)batch * h_kv * 4) + 255) / 256 * 256;
    e = cudaMemsetAsync(scratch, 0, ticket_bytes, s);
    if (e != cudaSuccess) return (int)e;
  }
  jssa::AttendArgs a = {};
  a.q = q; a.k_cache = k_cache; a.v_cache = v_cache;
  a.page_stride = kv_page_stride; a.slot_stride = kv_slot_stride; a.head_stride = kv_head_stride;
  a.block_table = block_table; a.max_pages = max_pages; a.idx = idx; a.count = count;
  a.batch = batch; a.h_q = h_q; a.h_kv = h_kv; a.d = d; a.budget = budget;
  a.num_pages = num_pages; a.page_size = page_size; a.scale = softmax_scale; a.out = out;
  a.ws = plan.ws_bytes ? scratch : nullptr;
  e = jssa::launch_attend(a, true, plan, false, s);
  return e == cudaSuccess ? JSSA_OK : (int)e;
}
