// pa_api.cu -- the C ABI of libpagedattn.so: argument validation, status and
// error messages, the TMA tensor-map cache and dispatch to the kernel launchers.
// Declarations and the contract of every entry point: include/pagedattn.h.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include "../../include/pagedattn.h"
#include "pa_internal.h"

namespace pa {

__device__ unsigned int g_watchdog = 0;

static thread_local std::string t_last_error;

// ------------------------------------------------- per-device launch state
namespace {
constexpr int kMaxDev = 64;
std::mutex g_dev_mu;
std::unordered_map<const void*, uint64_t> g_attr_done;   // kernel -> bitmask of devices
int g_sm_count[kMaxDev];
}  // namespace

pa_status ensure_smem_attr(const void* kernel, int bytes, const char* what) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const uint64_t bit = dev < kMaxDev ? (uint64_t)1 << dev : 0;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    auto it = g_attr_done.find(kernel);
    if (bit && it != g_attr_done.end() && (it->second & bit)) return PA_OK;
  }
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, what);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  g_attr_done[kernel] |= bit;
  return PA_OK;
}

void forget_smem_attr(const void* kernel) {
  std::lock_guard<std::mutex> lk(g_dev_mu);
  g_attr_done.erase(kernel);
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_sm_count[dev] > 0) return g_sm_count[dev];
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  g_sm_count[dev] = n;
  return n;
}

pa_status fail(pa_status s, const std::string& msg) {
  t_last_error = msg;
  return s;
}

pa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct MapKey {
  const void* base;
  int64_t rows;
  int heads, d;
  int64_t stride;
  int box, box_heads;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && heads == o.heads && d == o.d && stride == o.stride &&
           box == o.box && box_heads == o.box_heads;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = std::hash<const void*>()(k.base);
    h ^= std::hash<int64_t>()(k.rows * 1315423911ll + k.stride) + 0x9e3779b97f4a7c15ull + (h << 6);
    h ^= std::hash<int64_t>()((int64_t)k.heads << 40 | (int64_t)k.d << 20 | k.box) + (h << 6);
    h ^= std::hash<int>()(k.box_heads) + (h << 3);
    return h;
  }
};

static std::mutex g_map_mu;
static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;

pa_status get_tensor_map(CUtensorMap* out, const void* base, int64_t rows, int heads, int head_dim,
                         int64_t row_stride_elems, int box_rows, int box_heads) {
  MapKey key{base, rows, heads, head_dim, row_stride_elems, box_rows, box_heads};
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *out = it->second;
      return PA_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)row_stride_elems * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap m;
  CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof buf,
             "cuTensorMapEncodeTiled failed (%d) rows=%lld heads=%d d=%d box=%d x %d heads", (int)r,
             (long long)rows, heads, head_dim, box_rows, box_heads);
    return fail(PA_ERR_CUDA, buf);
  }
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    if (g_maps.size() > 512) g_maps.clear();
    g_maps.emplace(key, m);
  }
  *out = m;
  return PA_OK;
}

// ------------------------------------------------------------------ helpers
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

static pa_status check_common(const void* k_cache, const void* v_cache, int hq, int hkv, int d,
                              int block_size, int num_blocks, pa_dtype dtype) {
  if (dtype != PA_BF16) return fail(PA_ERR_UNSUPPORTED, "only PA_BF16 is implemented");
  if (!k_cache || !v_cache) return fail(PA_ERR_INVALID_ARG, "k_cache / v_cache is NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "k_cache / v_cache must be 16-byte aligned");
  if (hq <= 0 || hkv <= 0) return fail(PA_ERR_INVALID_ARG, "head counts must be positive");
  if (hq % hkv != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads must be a multiple of num_kv_heads");
  if (d != 64 && d != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (!pow2(block_size) || block_size < 16 || block_size > 1024)
    return fail(PA_ERR_UNSUPPORTED, "block_size must be a power of two in [16, 1024]");
  if (num_blocks <= 0) return fail(PA_ERR_INVALID_ARG, "num_blocks must be positive");
  if ((int64_t)num_blocks * block_size > INT32_MAX)
    return fail(PA_ERR_UNSUPPORTED, "num_blocks * block_size must fit in int32");
  return PA_OK;
}

int decode_auto_partition(int num_seqs, int num_kv_heads, int max_context_len) {
  // Aim for several waves of 2 CTAs per SM on a 148-SM part, with partitions
  // between 256 and 1024 tokens (64-token tiles).
  const int64_t target_ctas = 148 * 2 * 6;
  int64_t pairs = (int64_t)num_seqs * num_kv_heads;
  int64_t p = (pairs * (int64_t)max_context_len + target_ctas - 1) / target_ctas;
  p = (p + 63) / 64 * 64;
  if (p < 256) p = 256;
  if (p > 1024) p = 1024;
  return (int)p;
}

static void decode_ws_layout(int num_seqs, int hq, int d, int64_t splits, size_t* o_bytes,
                             size_t* ml_bytes) {
  size_t rows = (size_t)num_seqs * hq * splits;
  *o_bytes = (rows * d * sizeof(float) + 255) / 256 * 256;
  *ml_bytes = (rows * 2 * sizeof(float) + 255) / 256 * 256;
}

}  // namespace pa

using namespace pa;

// ====================================================================== C ABI
extern "C" {

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
  }
  return "PA_ERR_UNKNOWN";
}

const char* pa_last_error_message(void) { return t_last_error.c_str(); }

const char* pa_version(void) { return "pagedattn 0.1 sm_100a"; }

pa_status pa_store_kvcache(const void* key, const void* value, int64_t key_token_stride,
                           int64_t value_token_stride, void* k_cache, void* v_cache,
                           const int32_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                           int32_t head_dim, int64_t num_slots, pa_dtype dtype, int32_t* err_flag,
                           pa_stream_t stream) {
  t_last_error.clear();
  if (dtype != PA_BF16) return fail(PA_ERR_UNSUPPORTED, "only PA_BF16 is implemented");
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens < 0");
  if (num_kv_heads <= 0 || head_dim <= 0)
    return fail(PA_ERR_INVALID_ARG, "num_kv_heads and head_dim must be positive");
  int64_t row = (int64_t)num_kv_heads * head_dim;
  if (row % 8 != 0) return fail(PA_ERR_UNSUPPORTED, "num_kv_heads*head_dim must be a multiple of 8");
  if (key_token_stride < row || value_token_stride < row)
    return fail(PA_ERR_INVALID_ARG, "token stride smaller than num_kv_heads*head_dim");
  if (key_token_stride % 8 || value_token_stride % 8)
    return fail(PA_ERR_INVALID_ARG, "token strides must be multiples of 8 elements (16 bytes)");
  if (num_slots <= 0 || num_slots > INT32_MAX)
    return fail(PA_ERR_INVALID_ARG, "num_slots must be in [1, 2^31)");
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "key/value/k_cache/v_cache must be 16-byte aligned");
  return launch_store(key, value, key_token_stride, value_token_stride, k_cache, v_cache,
                      slot_mapping, num_tokens, (int)row, num_slots, err_flag,
                      (cudaStream_t)stream);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t max_context_len,
                                int32_t partition_size) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_context_len <= 0)
    return 0;
  int p = partition_size > 0 ? partition_size
                             : decode_auto_partition(num_seqs, num_kv_heads, max_context_len);
  if (p <= 0 || p % 64) return 0;
  const int64_t splits = ((int64_t)max_context_len + p - 1) / p;
  if (splits <= 1 || splits > 65535) return 0;
  size_t ob, mb;
  decode_ws_layout(num_seqs, num_q_heads, head_dim, splits, &ob, &mb);
  return ob + mb;
}

namespace {
struct FusedStore {
  const void* key;
  const void* value;
  int64_t key_stride, value_stride;
  const int32_t* slots;
};
}  // namespace

static pa_status decode_impl(void* out, const void* q, int64_t q_token_stride, const void* k_cache,
                             const void* v_cache, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                             int32_t num_seqs, int32_t max_context_len, int32_t num_q_heads,
                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                             int32_t num_blocks, float scale, int32_t partition_size,
                             void* workspace, size_t workspace_bytes, pa_dtype dtype,
                             int32_t* err_flag, pa_stream_t stream, const FusedStore* st) {
  pa_status s = check_common(k_cache, v_cache, num_q_heads, num_kv_heads, head_dim, block_size,
                             num_blocks, dtype);
  if (s != PA_OK) return s;
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "num_seqs < 0");
  if (num_seqs == 0) return PA_OK;
  if (num_seqs > 65535) return fail(PA_ERR_UNSUPPORTED, "num_seqs > 65535");
  if (!out || !q || !block_tables || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(out) || !aligned16(q)) return fail(PA_ERR_INVALID_ARG, "q/out must be 16-byte aligned");
  if (q_token_stride < (int64_t)num_q_heads * head_dim || q_token_stride % 8)
    return fail(PA_ERR_INVALID_ARG, "q_token_stride must be >= Hq*D and a multiple of 8");
  if (max_context_len <= 0) return fail(PA_ERR_INVALID_ARG, "max_context_len must be positive");
  if (max_blocks_per_seq <= 0) return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq must be positive");
  if ((int64_t)max_blocks_per_seq * block_size < max_context_len)
    return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq*block_size < max_context_len");
  if ((int64_t)num_blocks * block_size < max_context_len)
    return fail(PA_ERR_INVALID_ARG, "max_context_len exceeds the pool (num_blocks*block_size)");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (partition_size < 0 || partition_size % 64)
    return fail(PA_ERR_INVALID_ARG, "partition_size must be 0 (auto) or a positive multiple of 64");
  const int p = partition_size > 0 ? partition_size
                                   : decode_auto_partition(num_seqs, num_kv_heads, max_context_len);
  const int64_t splits64 = ((int64_t)max_context_len + p - 1) / p;
  if (splits64 > 65535) return fail(PA_ERR_UNSUPPORTED, "too many partitions; raise partition_size");
  const int splits = (int)splits64;
  DecodeArgs a{};
  a.out = out; a.q = q; a.q_stride = q_token_stride;
  a.k_cache = k_cache; a.v_cache = v_cache;
  a.block_tables = block_tables; a.max_blocks = max_blocks_per_seq;
  a.context_lens = context_lens; a.num_seqs = num_seqs; a.max_context_len = max_context_len;
  a.hq = num_q_heads; a.hkv = num_kv_heads; a.d = head_dim;
  a.block_size = block_size; a.num_blocks = num_blocks; a.scale = scale;
  a.partition = p; a.max_splits = splits;
  a.err_flag = err_flag; a.stream = (cudaStream_t)stream;
  if (splits > 1) {
    size_t ob, mb;
    decode_ws_layout(num_seqs, num_q_heads, head_dim, splits, &ob, &mb);
    if (!workspace || workspace_bytes < ob + mb) {
      char buf[128];
      snprintf(buf, sizeof buf, "workspace of %zu bytes needed (%d partitions), got %zu", ob + mb,
               splits, workspace_bytes);
      return fail(PA_ERR_WORKSPACE, buf);
    }
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
      return fail(PA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    a.ws_o = static_cast<float*>(workspace);
    a.ws_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + ob);
  }
  if (st) {
    a.new_k = st->key;
    a.new_v = st->value;
    a.new_k_stride = st->key_stride;
    a.new_v_stride = st->value_stride;
    a.slots = st->slots;
  }
  return launch_decode(a);
}

pa_status pa_decode(void* out, const void* q, int64_t q_token_stride, const void* k_cache,
                    const void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t num_seqs, int32_t max_context_len,
                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                    int32_t block_size, int32_t num_blocks, float scale, int32_t partition_size,
                    void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* err_flag,
                    pa_stream_t stream) {
  t_last_error.clear();
  return decode_impl(out, q, q_token_stride, k_cache, v_cache, block_tables, max_blocks_per_seq,
                     context_lens, num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                     block_size, num_blocks, scale, partition_size, workspace, workspace_bytes,
                     dtype, err_flag, stream, nullptr);
}

pa_status pa_decode_store(void* out, const void* q, int64_t q_token_stride, const void* key,
                          const void* value, int64_t key_token_stride, int64_t value_token_stride,
                          const int32_t* slot_mapping, void* k_cache, void* v_cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                          const int32_t* context_lens, int32_t num_seqs, int32_t max_context_len,
                          int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t block_size, int32_t num_blocks, float scale,
                          int32_t partition_size, void* workspace, size_t workspace_bytes,
                          pa_dtype dtype, int32_t* err_flag, pa_stream_t stream) {
  t_last_error.clear();
  if (num_seqs > 0) {
    if (!key || !value || !slot_mapping) return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned16(key) || !aligned16(value))
      return fail(PA_ERR_INVALID_ARG, "key/value must be 16-byte aligned");
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (key_token_stride < row || value_token_stride < row)
      return fail(PA_ERR_INVALID_ARG, "token stride smaller than num_kv_heads*head_dim");
    if (key_token_stride % 8 || value_token_stride % 8)
      return fail(PA_ERR_INVALID_ARG, "token strides must be multiples of 8 elements (16 bytes)");
  }
  const FusedStore st{key, value, key_token_stride, value_token_stride, slot_mapping};
  return decode_impl(out, q, q_token_stride, k_cache, v_cache, block_tables, max_blocks_per_seq,
                     context_lens, num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                     block_size, num_blocks, scale, partition_size, workspace, workspace_bytes,
                     dtype, err_flag, stream, &st);
}

// Validation and launch shared by pa_prefill_varlen and pa_prefill_store
// (fused store when a.slot_mapping is set).
static pa_status prefill_entry(PrefillArgs& a, void* out, const void* q, int64_t q_token_stride,
                               const void* k_cache, const void* v_cache,
                               const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                               int32_t max_seqlen_q, int32_t max_seqlen_k, int32_t total_q,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t num_blocks,
                               float scale, pa_dtype dtype, int32_t* err_flag,
                               pa_stream_t stream) {
  pa_status s = check_common(k_cache, v_cache, num_q_heads, num_kv_heads, head_dim, block_size,
                             num_blocks, dtype);
  if (s != PA_OK) return s;
  if (num_seqs < 0 || total_q < 0) return fail(PA_ERR_INVALID_ARG, "num_seqs / total_q < 0");
  if (num_seqs == 0 || total_q == 0) return PA_OK;
  if (num_seqs > 65535) return fail(PA_ERR_UNSUPPORTED, "num_seqs > 65535");
  if (!out || !q || !cu_seqlens_q || !cu_seqlens_k || !block_tables)
    return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
  if (!aligned16(out) || !aligned16(q)) return fail(PA_ERR_INVALID_ARG, "q/out must be 16-byte aligned");
  if (q_token_stride < (int64_t)num_q_heads * head_dim || q_token_stride % 8)
    return fail(PA_ERR_INVALID_ARG, "q_token_stride must be >= Hq*D and a multiple of 8");
  if (max_seqlen_q <= 0 || max_seqlen_k < max_seqlen_q)
    return fail(PA_ERR_INVALID_ARG, "need 0 < max_seqlen_q <= max_seqlen_k");
  if (max_blocks_per_seq <= 0 || (int64_t)max_blocks_per_seq * block_size < max_seqlen_k)
    return fail(PA_ERR_INVALID_ARG, "max_blocks_per_seq*block_size < max_seqlen_k");
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (a.slot_mapping) {
    if (!a.key || !a.value) return fail(PA_ERR_INVALID_ARG, "key / value is NULL");
    if (!aligned16(a.key) || !aligned16(a.value))
      return fail(PA_ERR_INVALID_ARG, "key / value must be 16-byte aligned");
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (a.key_stride < row || a.value_stride < row || a.key_stride % 8 || a.value_stride % 8)
      return fail(PA_ERR_INVALID_ARG, "key/value token strides must be >= Hkv*D and multiples of 8");
  }
  a.out = out; a.q = q; a.q_stride = q_token_stride; a.total_q = total_q;
  a.k_cache = k_cache; a.v_cache = v_cache; a.cu_q = cu_seqlens_q; a.cu_k = cu_seqlens_k;
  a.max_seqlen_q = max_seqlen_q; a.max_seqlen_k = max_seqlen_k;
  a.block_tables = block_tables; a.max_blocks = max_blocks_per_seq; a.num_seqs = num_seqs;
  a.hq = num_q_heads; a.hkv = num_kv_heads; a.d = head_dim;
  a.block_size = block_size; a.num_blocks = num_blocks; a.scale = scale;
  a.err_flag = err_flag; a.stream = (cudaStream_t)stream;
  return launch_prefill(a);
}

pa_status pa_prefill_varlen(void* out, const void* q, int64_t q_token_stride, const void* k_cache,
                            const void* v_cache, const int32_t* cu_seqlens_q,
                            const int32_t* cu_seqlens_k, int32_t max_seqlen_q,
                            int32_t max_seqlen_k, int32_t total_q, const int32_t* block_tables,
                            int32_t max_blocks_per_seq, int32_t num_seqs, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int32_t num_blocks, float scale, pa_dtype dtype, int32_t* err_flag,
                            pa_stream_t stream) {
  t_last_error.clear();
  PrefillArgs a{};
  return prefill_entry(a, out, q, q_token_stride, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k,
                       max_seqlen_q, max_seqlen_k, total_q, block_tables, max_blocks_per_seq,
                       num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       scale, dtype, err_flag, stream);
}

pa_status pa_prefill_store(void* out, const void* q, int64_t q_token_stride, const void* key,
                           const void* value, int64_t key_token_stride,
                           int64_t value_token_stride, const int32_t* slot_mapping, void* k_cache,
                           void* v_cache, const int32_t* cu_seqlens_q,
                           const int32_t* cu_seqlens_k, int32_t max_seqlen_q,
                           int32_t max_seqlen_k, int32_t total_q, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, int32_t num_seqs, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           int32_t num_blocks, float scale, pa_dtype dtype, int32_t* err_flag,
                           pa_stream_t stream) {
  t_last_error.clear();
  if (!slot_mapping) return fail(PA_ERR_INVALID_ARG, "slot_mapping is NULL");
  PrefillArgs a{};
  a.key = key;
  a.value = value;
  a.key_stride = key_token_stride;
  a.value_stride = value_token_stride;
  a.slot_mapping = slot_mapping;
  return prefill_entry(a, out, q, q_token_stride, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k,
                       max_seqlen_q, max_seqlen_k, total_q, block_tables, max_blocks_per_seq,
                       num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                       scale, dtype, err_flag, stream);
}

pa_status pa_watchdog_read(uint32_t* value) {
  t_last_error.clear();
  if (!value) return fail(PA_ERR_INVALID_ARG, "value is NULL");
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_watchdog, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e, "reading the watchdog word");
  e = cudaMemcpyToSymbol(g_watchdog, &zero, sizeof zero);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the watchdog word");
  *value = v;
  return PA_OK;
}

}  // extern "C"
