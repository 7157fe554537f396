// store_kvcache.cu -- scatter each step's new K/V rows into the paged pool.
//
// "Deep into the Nano-vLLM inference engine" (lnwmold.com), sections "From
// Sequences to Blocks" and "Control plane vs. data plane": every token of a
// sequence has a place (slot) in a fixed-size block chosen by the CPU block
// manager; the GPU side only moves the data.  Slot s is flat token row s of
// the [num_blocks * block_size, Hkv, D] view of each pool; slot < 0 = skip.
//
// HBM-bound copy: each 16-byte chunk of a row is read once with a
// non-allocating vector load and written once with a vector store.  A CTA of
// 256 threads covers ROWS whole rows (row = Hkv*D bf16) for both K and V, so
// consecutive threads touch consecutive 16-byte chunks of the same row.

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(256) store_kvcache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, int64_t key_stride16,
    int64_t value_stride16, uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
    const int32_t* __restrict__ slots, int num_tokens, int row16, int rows_per_cta,
    int64_t num_slots, int32_t* err_flag) {
  pdl_wait();
  pdl_trigger();
  // thread -> (row within the CTA, first chunk); long rows are strided by the CTA
  const bool long_row = row16 >= (int)blockDim.x;
  const int lr = long_row ? 0 : (int)threadIdx.x / row16;
  const int c0 = long_row ? (int)threadIdx.x : (int)threadIdx.x % row16;
  const int step = long_row ? (int)blockDim.x : row16;
  if (lr >= rows_per_cta) return;
  const int64_t tok = (int64_t)blockIdx.x * rows_per_cta + lr;
  if (tok >= num_tokens) return;
  const int32_t slot = __ldg(slots + tok);
  if (slot < 0) return;
  if ((int64_t)slot >= num_slots) {
    if (c0 == 0) raise_flag(err_flag, PA_FLAG_SLOT_OOB);
    return;
  }
  for (int c = c0; c < row16; c += step) {
    uint4 kv = ld_stream(key + tok * key_stride16 + c);
    uint4 vv = ld_stream(value + tok * value_stride16 + c);
    k_cache[(int64_t)slot * row16 + c] = kv;
    v_cache[(int64_t)slot * row16 + c] = vv;
  }
}

pa_status launch_store(const void* key, const void* value, int64_t key_stride,
                       int64_t value_stride, void* k_cache, void* v_cache, const int32_t* slots,
                       int num_tokens, int row_elems, int64_t num_slots, int32_t* err_flag,
                       cudaStream_t stream) {
  const int row16 = row_elems / 8;
  const int threads = 256;
  // rows per CTA: fill the CTA when rows are short, one row otherwise
  int rows_per_cta = row16 >= threads ? 1 : threads / row16;
  int64_t grid = (num_tokens + rows_per_cta - 1) / rows_per_cta;
  if (grid > INT32_MAX) return fail(PA_ERR_UNSUPPORTED, "too many tokens");
  cudaError_t e = launch_pdl(store_kvcache_kernel, dim3((unsigned)grid), dim3(threads), 0, stream,
                             static_cast<const uint4*>(key), static_cast<const uint4*>(value),
                             key_stride / 8, value_stride / 8, static_cast<uint4*>(k_cache),
                             static_cast<uint4*>(v_cache), slots, num_tokens, row16, rows_per_cta,
                             num_slots, err_flag);
  if (e != cudaSuccess) return cuda_fail(e, "store_kvcache launch");
  return PA_OK;
}

}  // namespace pa
