// prefill_tc.cu -- varlen causal prefill over the paged pool on the 5th-gen
// tensor cores (tcgen05 + TMEM), head_dim 128.
//
// Definition (same as prefill_mma.cu): sequence i computes q_len new queries
// over k_len keys, the first k_len - q_len a cached prefix shared through the
// hash prefix cache ("Prefix Caching via hashing", lnwmold.com item); query j
// attends keys 0 .. k_len-q_len+j; prompts are batched by cumulative sequence
// lengths ("Preparation before computation", same item).
//
// One CTA = 128 query rows of one (sequence, query head); 6 warps:
//   warp 4      TMA producer: the Q tile once, then 128-key K and V tiles of
//               the sequence (one box per physical block chunk, 128-byte
//               swizzle) into a 2-stage ring; zeroes V rows of the last tile
//               past the CTA's last visible key (stale rows may be NaN).
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM S
//               buffers (M=128, N=128, K=16 x 8), then O += P_j V_j into the
//               TMEM O accumulator (A = P from shared memory, B = V MN-major);
//               tcgen05.commit signals mbarriers.  S_{j+1} is issued before
//               waiting for P_j, so QK^T of the next tile overlaps the softmax.
//   warps 0-3   softmax, one thread per query row (TMEM lane): tcgen05.ld the
//               S row, causal mask, online softmax in the log2 domain with a
//               lazy rescale (the reference max moves only when it grows by
//               more than 8, i.e. a factor 256), P as bf16 into shared memory
//               (swizzled, K-major), O rescaled in TMEM when needed; epilogue
//               O / l -> bf16 -> global.
// TMEM: 512 columns (S0 | S1 | O | unused).  Shared memory: Q 32 KB, K and V
// 2 x 32 KB each, P 32 KB.  Every wait is bounded; an abort winds all roles
// down, drains the issued MMAs and frees TMEM.

#include <cmath>

#include "pa_common.cuh"
#include "pa_internal.h"
#include "tc_common.cuh"

namespace pa {

constexpr int kTcRows = 128;     // query rows per CTA (MMA M)
constexpr int kTcKeys = 128;     // keys per tile (MMA N of QK^T, K of PV)
constexpr int kTcThreads = 192;
constexpr int kTile = 32768;     // one 128 x 128 bf16 operand: two 128 x 64 swizzled halves
constexpr int kHalf = 16384;
constexpr float kLazyRescale = 8.f;   // log2 of the largest un-rescaled growth (256x)

struct PrefillTcParams {
  __nv_bfloat16* out;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* block_tables;
  int max_blocks;
  int hq, group;
  int block_size, log2_bs, box_rows;
  int num_blocks, num_slots;
  int max_seqlen_q, max_seqlen_k, total_q;
  float scale_log2;
  int32_t* err_flag;
};

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        int32_t* err_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        raise_flag(err_flag, PA_FLAG_TIMEOUT);
        return false;
      }
    }
  }
}

__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kTile;              // [2 stages]
  uint8_t* sV = sK + 2 * kTile;          // [2 stages]
  uint8_t* sP = sV + 2 * kTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + kTile);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;           // [2]
  uint64_t* v_full = bars + 3;           // [2]
  uint64_t* kv_empty = bars + 5;         // [2]
  uint64_t* s_full = bars + 7;           // [2]
  uint64_t* s_free = bars + 9;           // [2]
  uint64_t* p_full = bars + 11;
  uint64_t* pv_done = bars + 12;
  uint64_t* vz_ready = bars + 13;
  uint64_t* drain = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 16);

  const int qtile = blockIdx.x, h = blockIdx.y, seq = blockIdx.z;
  const int kvh = h / p.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // sequence bounds
  const int cq0 = __ldg(p.cu_q + seq), cq1 = __ldg(p.cu_q + seq + 1);
  const int ck0 = __ldg(p.cu_k + seq), ck1 = __ldg(p.cu_k + seq + 1);
  const int q_start = cq0, q_len = cq1 - cq0, k_len = ck1 - ck0;
  if (!(cq0 >= 0 && q_len >= 0 && cq1 <= p.total_q && k_len >= q_len &&
        q_len <= p.max_seqlen_q && k_len <= p.max_seqlen_k && k_len <= p.max_blocks * p.block_size)) {
    if (threadIdx.x == 0 && qtile == 0 && h == 0) raise_flag(p.err_flag, PA_FLAG_LEN_OOB);
    return;
  }
  const int q0 = qtile * kTcRows;
  if (q0 >= q_len) return;
  const int cached = k_len - q_len;
  const int kv_end = min(k_len, cached + min(q_len, q0 + kTcRows));   // keys any row can see
  const int n = (kv_end + kTcKeys - 1) / kTcKeys;
  const int last_valid = kv_end - (n - 1) * kTcKeys;
  const bool zero_tail = last_valid < kTcKeys;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(vz_ready, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;               // S buffers: columns [0,128) and [128,256)
  const uint32_t tO = tmem + 256;         // O accumulator: columns [256,384)

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, kTile);
      tma_load_3d(sQ, &tmQ, q_full, 0, h, q_start + q0);
      tma_load_3d(sQ + kHalf, &tmQ, q_full, 64, h, q_start + q0);
      const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks;
      const int box = p.box_rows;
      for (int j = 0; j < n; ++j) {
        const int st = j & 1;
        if (j >= 2 && !tc_wait(&kv_empty[st], ((j >> 1) - 1) & 1, abort_flag, p.err_flag)) break;
        const int t0 = j * kTcKeys;
        const int nbox = (min(kTcKeys, kv_end - t0) + box - 1) / box;
        const uint32_t bytes = (uint32_t)(nbox * box * 128 * 2);
        int rows[kTcKeys / 16];
        for (int b = 0; b < nbox; ++b) {
          const int t = t0 + b * box;
          const int bid = __ldg(bt + (t >> p.log2_bs));
          if (bid < 0 || bid >= p.num_blocks) {
            raise_flag(p.err_flag, PA_FLAG_BLOCK_OOB);
            rows[b] = p.num_slots;                 // past the pool: TMA fills zeros
          } else {
            rows[b] = bid * p.block_size + (t & (p.block_size - 1));
          }
        }
        mbar_arrive_expect_tx(&k_full[st], bytes);
        for (int b = 0; b < nbox; ++b) {
          uint8_t* dst = sK + st * kTile + b * box * 128;
          tma_load_3d(dst, &tmK, &k_full[st], 0, kvh, rows[b]);
          tma_load_3d(dst + kHalf, &tmK, &k_full[st], 64, kvh, rows[b]);
        }
        mbar_arrive_expect_tx(&v_full[st], bytes);
        for (int b = 0; b < nbox; ++b) {
          uint8_t* dst = sV + st * kTile + b * box * 128;
          tma_load_3d(dst, &tmV, &v_full[st], 0, kvh, rows[b]);
          tma_load_3d(dst + kHalf, &tmV, &v_full[st], 64, kvh, rows[b]);
        }
      }
    }
    __syncwarp();
    if (zero_tail) {
      const int j = n - 1, st = j & 1;
      if (tc_wait(&v_full[st], (j >> 1) & 1, abort_flag, p.err_flag)) {
        const int nrow = kTcKeys - last_valid;
        for (int i = lane; i < nrow * 16; i += 32) {
          const int hf = i / (nrow * 8);
          const int rr = (i / 8) % nrow;
          *reinterpret_cast<uint4*>(sV + st * kTile + hf * kHalf + (last_valid + rr) * 128 +
                                    (i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(vz_ready);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(kTcRows, kTcKeys, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(kTcRows, 128, false, true);
      const uint32_t aQ = smem_u32(sQ), aP = smem_u32(sP);
      bool ok = tc_wait(q_full, 0, abort_flag, p.err_flag);
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!tc_wait(&k_full[st], (j >> 1) & 1, abort_flag, p.err_flag)) return false;
        if (j >= 2 && !tc_wait(&s_free[st], ((j >> 1) - 1) & 1, abort_flag, p.err_flag)) return false;
        tc::fence_after_sync();
        const uint32_t aK = smem_u32(sK + st * kTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t o = (ks >> 2) * kHalf + (ks & 3) * 32;
          tc::mma_ss(tS + st * 128, tc::sdesc_sw128(aQ + o, 16, 1024),
                     tc::sdesc_sw128(aK + o, 16, 1024), idS, ks > 0);
        }
        tc::commit(&s_full[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n && !issue_s(j + 1)) break;
        if (!tc_wait(p_full, j & 1, abort_flag, p.err_flag)) break;
        const bool vz = zero_tail && j == n - 1;
        if (!tc_wait(vz ? vz_ready : &v_full[j & 1], vz ? 0u : (uint32_t)((j >> 1) & 1), abort_flag,
                     p.err_flag))
          break;
        tc::fence_after_sync();
        const uint32_t aV = smem_u32(sV + (j & 1) * kTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t oa = (ks >> 2) * kHalf + (ks & 3) * 32;
          tc::mma_ss(tO, tc::sdesc_sw128(aP + oa, 16, 1024),
                     tc::sdesc_sw128(aV + ks * 2048, kHalf, 1024), idO, (j > 0 || ks > 0));
        }
        tc::commit(pv_done);
        tc::commit(&kv_empty[j & 1]);
      }
      // every issued MMA finishes before TMEM is released
      tc::commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;                         // query row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int limit = min(cached + q0 + r, k_len - 1);  // last visible key of this row
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t sv[kTcKeys];
    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      if (!tc_wait(&s_full[b], (j >> 1) & 1, abort_flag, p.err_flag)) { ok = false; break; }
      tc::fence_after_sync();
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::ld32(tS + lane_off + b * 128 + c * 32, sv + c * 32);
      tc::wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);
      const int t0 = j * kTcKeys;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kTcKeys; ++i) {
        const float s = (t0 + i <= limit) ? __uint_as_float(sv[i]) * p.scale_log2 : -INFINITY;
        sv[i] = __float_as_uint(s);
        mx = fmaxf(mx, s);
      }
      float alpha = 1.f;
      bool resc = false;
      if (m_ref == -INFINITY) {
        m_ref = mx;                                    // first tile with a visible key
      } else if (mx > m_ref + kLazyRescale) {
        alpha = fast_exp2(m_ref - mx);
        m_ref = mx;
        resc = true;
        l *= alpha;
      }
      const float mref = m_ref == -INFINITY ? 0.f : m_ref;
      float rs = 0.f;
#pragma unroll
      for (int i = 0; i < kTcKeys; ++i) {
        const float e = fast_exp2(__uint_as_float(sv[i]) - mref);
        rs += e;
        sv[i] = __float_as_uint(e);
      }
      l += rs;
      // PV_{j-1} must be done before P is overwritten and O is rescaled
      if (j > 0 && !tc_wait(pv_done, (j - 1) & 1, abort_flag, p.err_flag)) { ok = false; break; }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const int i0 = hf * 64 + ch * 8;
          uint4 v;
          v.x = pack_bf16(__uint_as_float(sv[i0 + 0]), __uint_as_float(sv[i0 + 1]));
          v.y = pack_bf16(__uint_as_float(sv[i0 + 2]), __uint_as_float(sv[i0 + 3]));
          v.z = pack_bf16(__uint_as_float(sv[i0 + 4]), __uint_as_float(sv[i0 + 5]));
          v.w = pack_bf16(__uint_as_float(sv[i0 + 6]), __uint_as_float(sv[i0 + 7]));
          *reinterpret_cast<uint4*>(sP + hf * kHalf + sw128(r, ch)) = v;
        }
      if (__any_sync(0xffffffffu, resc)) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tc::ld32(tO + lane_off + c * 32, ov);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tc::st32(tO + lane_off + c * 32, ov);
        }
        tc::wait_st();
      }
      fence_proxy_async_smem();                        // P visible to the tensor core
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // epilogue: O / l -> bf16
    if (ok && tc_wait(pv_done, (n - 1) & 1, abort_flag, p.err_flag)) {
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool store = q0 + r < q_len;
      __nv_bfloat16* orow = p.out + ((int64_t)(q_start + q0 + r) * p.hq + h) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tc::ld32(tO + lane_off + c * 32, ov);
        tc::wait_ld();
        if (store) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(ov[8 * k + 0]) * inv, __uint_as_float(ov[8 * k + 1]) * inv);
            v.y = pack_bf16(__uint_as_float(ov[8 * k + 2]) * inv, __uint_as_float(ov[8 * k + 3]) * inv);
            v.z = pack_bf16(__uint_as_float(ov[8 * k + 4]) * inv, __uint_as_float(ov[8 * k + 5]) * inv);
            v.w = pack_bf16(__uint_as_float(ov[8 * k + 6]) * inv, __uint_as_float(ov[8 * k + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + c * 32 + k * 8) = v;
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

pa_status launch_prefill_tc(const PrefillArgs& a) {
  const int box = a.block_size < kTcKeys ? a.block_size : kTcKeys;
  const int64_t slots = (int64_t)a.num_blocks * a.block_size;
  CUtensorMap mq, mk, mv;
  pa_status s = get_tensor_map(&mq, a.q, a.total_q, a.hq, a.d, a.q_stride, kTcRows);
  if (s != PA_OK) return s;
  s = get_tensor_map(&mk, a.k_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  s = get_tensor_map(&mv, a.v_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  PrefillTcParams prm{};
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.cu_q = a.cu_q;
  prm.cu_k = a.cu_k;
  prm.block_tables = a.block_tables;
  prm.max_blocks = a.max_blocks;
  prm.hq = a.hq;
  prm.group = a.hq / a.hkv;
  prm.block_size = a.block_size;
  prm.log2_bs = __builtin_ctz((unsigned)a.block_size);
  prm.box_rows = box;
  prm.num_blocks = a.num_blocks;
  prm.num_slots = (int)slots;
  prm.max_seqlen_q = a.max_seqlen_q;
  prm.max_seqlen_k = a.max_seqlen_k;
  prm.total_q = a.total_q;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.err_flag = a.err_flag;
  const size_t smem = 6 * (size_t)kTile + 1024 + 256;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "prefill_tc smem attribute");
    attr_done = true;
  }
  if (a.hq > 65535) return fail(PA_ERR_UNSUPPORTED, "too many heads");
  dim3 grid((a.max_seqlen_q + kTcRows - 1) / kTcRows, a.hq, a.num_seqs);
  prefill_tc_kernel<<<grid, kTcThreads, smem, a.stream>>>(mq, mk, mv, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prefill_tc launch");
  return PA_OK;
}

}  // namespace pa
