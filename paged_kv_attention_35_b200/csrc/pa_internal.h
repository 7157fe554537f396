// pa_internal.h -- host-side pieces shared by the library's translation units:
// the thread-local error message, TMA tensor-map encoding for the KV pools, and
// the kernel launchers behind the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <utility>

#include "../../include/pagedattn.h"

namespace pa {

// Launches `kern` on `stream` with programmatic stream serialization allowed:
// the kernels call pdl_wait() before reading inputs, so a launch may be
// scheduled while the previous kernel on the stream drains.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device.  The attribute belongs to the device's context, so it is set once
// per device (and again after a context is re-created: a launch that fails
// with too little shared memory clears the record).
pa_status ensure_smem_attr(const void* kernel, int bytes, const char* what);
void forget_smem_attr(const void* kernel);

// Number of SMs of the current device (cached per device).
int device_sm_count();

// Records `msg` as this thread's last error and returns `s`.
pa_status fail(pa_status s, const std::string& msg);
pa_status cuda_fail(cudaError_t e, const char* what);

// A 3-D view [rows, heads, head_dim] of a bf16 buffer (a KV pool or packed q)
// as a TMA tensor map with 128-byte swizzle and boxes of {64, box_heads,
// box_rows}.  Cached per (pointer, shape, box); thread-safe.  Fills *out on
// success.
pa_status get_tensor_map(CUtensorMap* out, const void* base, int64_t rows, int heads, int head_dim,
                         int64_t row_stride_elems, int box_rows, int box_heads = 1);

struct DecodeArgs {
  void* out;
  const void* q;
  int64_t q_stride;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  int num_seqs;
  int max_context_len;
  int hq, hkv, d, block_size, num_blocks;
  float scale;
  int partition;       // tokens per partition (multiple of 64)
  int max_splits;      // ceil(max_context_len / partition)
  float* ws_o;         // [B, Hq, max_splits, D]
  float* ws_ml;        // [B, Hq, max_splits, 2]
  // fused store (pa_decode_store): row i of new_k / new_v goes to pool slot
  // slots[i] before attention; null slots = plain decode
  const void* new_k;
  const void* new_v;
  int64_t new_k_stride, new_v_stride;   // elements between tokens
  const int32_t* slots;
  int32_t* err_flag;
  cudaStream_t stream;
};

int decode_auto_partition(int num_seqs, int num_kv_heads, int max_context_len);
pa_status launch_decode(const DecodeArgs& a);

pa_status launch_store(const void* key, const void* value, int64_t key_stride,
                       int64_t value_stride, void* k_cache, void* v_cache,
                       const int32_t* slots, int num_tokens, int row_elems, int64_t num_slots,
                       int32_t* err_flag, cudaStream_t stream);

struct PrefillArgs {
  void* out;
  const void* q;
  int64_t q_stride;
  int total_q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int max_seqlen_q, max_seqlen_k;
  const int32_t* block_tables;
  int max_blocks;
  int num_seqs;
  int hq, hkv, d, block_size, num_blocks;
  float scale;
  int32_t* err_flag;
  cudaStream_t stream;
  // fused store (slot_mapping != nullptr): the batch's new K/V rows, written
  // to the pool by the same launch and read by attention from these arrays
  const void* key = nullptr;
  const void* value = nullptr;
  int64_t key_stride = 0, value_stride = 0;   // elements between tokens
  const int32_t* slot_mapping = nullptr;
};

pa_status launch_prefill(const PrefillArgs& a);

}  // namespace pa
