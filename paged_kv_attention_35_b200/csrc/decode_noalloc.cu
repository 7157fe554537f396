// decode_noalloc.cu -- pa_decode_noalloc: paged decode for callers that cannot
// allocate device memory themselves.
//
// pa_decode needs a caller-provided workspace for its split-K partials.  Some
// callers have no way to provide one: a serving engine that reserves all of
// the GPU's memory for its KV pool and activations at start-up and must not
// call cudaMalloc later (the call could fail once the pool owns the memory,
// and cudaFree synchronises the whole device), or a plain C host program that
// links only this library and receives its q / pool / output buffers ready
// made from another component, with no allocator of its own.  For them this
// entry point uses a fixed scratch array that belongs to the library: a
// file-scope static __device__ array of PA_DECODE_NOALLOC_SCRATCH_BYTES, which
// every GPU that loads the library holds until the process exits.
//
// Host code cannot use the array's name as a device address (in host code it
// is only a stand-in symbol), so the first call in each CUDA context -- once
// per device, with that device current -- asks the runtime for the array's
// device address (cudaGetSymbolAddress) and remembers it together with the
// context's unique id; a call from a context re-created since (after
// cudaDeviceReset, say) finds a different id and looks the address up again.
// After that the call is pa_decode with the scratch in place of the caller's
// workspace.  All calls share the one array and it keeps whatever the last
// call left in it: nothing there has to start at zero (the decode writes every
// partial before its merge reads it), but calls that overlap on the GPU -- two
// streams, or two host threads launching at once -- race on it.

#include <mutex>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[PA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
struct ScratchAddr {
  unsigned long long ctx_id;   // cuCtxGetId of the context the address belongs to
  void* addr;                  // device address of g_decode_scratch there
};
ScratchAddr g_scratch[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
      get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// Device address of the scratch array in the current device's context.
pa_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_UNSUPPORTED, "device ordinal >= 64");
  // 0 when no context is current yet: the lookup below then makes the
  // device's primary context current, and its id is read afterwards
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchAddr& c = g_scratch[dev];
  if (c.addr == nullptr || ctx == 0 || c.ctx_id != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
    if (p == nullptr) return fail(PA_ERR_CUDA, "cudaGetSymbolAddress returned NULL");
    c.addr = p;
    c.ctx_id = ctx ? ctx : current_context_id();
  }
  *out = c.addr;
  return PA_OK;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, int64_t q_token_stride,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                                       const int32_t* context_lens, int32_t num_seqs,
                                       int32_t max_context_len, int32_t num_q_heads,
                                       int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                       int32_t num_blocks, float scale, int32_t partition_size,
                                       pa_dtype dtype, int32_t* err_flag, pa_stream_t stream) {
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               max_context_len, partition_size);
  if (need > (size_t)PA_DECODE_NOALLOC_SCRATCH_BYTES) {
    char buf[200];
    snprintf(buf, sizeof buf,
             "pa_decode_noalloc: these sizes need %zu bytes of split-K scratch, more than the "
             "library's fixed %u bytes; use a larger partition_size or pa_decode with a workspace",
             need, (unsigned)PA_DECODE_NOALLOC_SCRATCH_BYTES);
    return fail(PA_ERR_WORKSPACE, buf);
  }
  void* scratch = nullptr;
  if (need > 0) {
    pa_status s = scratch_address(&scratch);
    if (s != PA_OK) return s;
  }
  return pa_decode(out, q, q_token_stride, k_cache, v_cache, block_tables, max_blocks_per_seq,
                   context_lens, num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                   block_size, num_blocks, scale, partition_size, scratch,
                   need > 0 ? (size_t)PA_DECODE_NOALLOC_SCRATCH_BYTES : 0, dtype, err_flag, stream);
}
