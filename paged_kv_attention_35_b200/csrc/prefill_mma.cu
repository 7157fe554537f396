// prefill_mma.cu -- varlen causal prefill over the paged pool, mma.sync path.
//
// Definition: sequence i computes q_len = cu_q[i+1]-cu_q[i] new queries over
// k_len = cu_k[i+1]-cu_k[i] keys, the first k_len-q_len of them a cached
// prefix reused through the hash prefix cache ("Prefix Caching via hashing",
// lnwmold.com item); query j attends keys 0 .. k_len-q_len+j (bottom-right
// causal alignment), softmax(scale q.k) v as in decode.  Cumulative sequence
// lengths batch the prompts ("Preparation before computation", same item).
//
// Design: grid (64-row query tile, query head, sequence).  One producer warp
// streams 64-token K/V tiles of the sequence from the pool with TMA (same
// tensor maps and boxes as decode) into a 3-stage ring; four consumer warps
// own 16 query rows each and run every KV tile up to the tile's causal limit:
// S = Q K^T and O += P V with mma.sync m16n8k16 (bf16 in, fp32 accumulate),
// online softmax in the log2 domain.  This path serves head_dim 64 and is
// the portable reference kernel for head_dim 128; the tcgen05/TMEM kernel in
// prefill_tc.cu is the fast path for head_dim 128.

#include <cmath>
#include <cstdlib>
#include <cstring>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kPfTile = 64;      // keys per pipeline stage and query rows per CTA
constexpr int kPfWarps = 4;
constexpr int kPfThreads = (kPfWarps + 1) * 32;
constexpr int kPfStages = 3;

struct PrefillMmaParams {
  const __nv_bfloat16* q;
  int64_t q_stride;
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

__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
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

// Reads the sequence's bounds; returns false (and flags) when they are inconsistent.
__device__ __forceinline__ bool seq_bounds(const PrefillMmaParams& p, int seq, int& q_start,
                                           int& q_len, int& k_len) {
  const int q0 = __ldg(p.cu_q + seq), q1 = __ldg(p.cu_q + seq + 1);
  const int k0 = __ldg(p.cu_k + seq), k1 = __ldg(p.cu_k + seq + 1);
  q_start = q0;
  q_len = q1 - q0;
  k_len = k1 - k0;
  const bool ok = q0 >= 0 && q_len >= 0 && q1 <= p.total_q && k_len >= q_len &&
                  q_len <= p.max_seqlen_q && k_len <= p.max_seqlen_k &&
                  k_len <= p.max_blocks * p.block_size;
  return ok;
}

template <int D, int STAGES>
__global__ void __launch_bounds__(kPfThreads, 2)
    prefill_mma_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const PrefillMmaParams p) {
  constexpr int HALVES = D / 64;
  constexpr int HALF_BYTES = kPfTile * 128;
  constexpr int KV_BYTES = HALVES * HALF_BYTES;
  constexpr int STAGE_BYTES = 2 * KV_BYTES;
  constexpr int KSTEPS = D / 16;
  constexpr int NT_O = D / 8;
  constexpr int NT_S = kPfTile / 8;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* ready = empty + STAGES;                // last tile zeroed (see below)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ready + 1);

  pdl_wait();
  pdl_trigger();
  const int qtile = blockIdx.x;
  const int h = blockIdx.y;
  const int seq = blockIdx.z;
  const int kvh = h / p.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int q_start, q_len, k_len;
  if (!seq_bounds(p, seq, q_start, q_len, k_len)) {
    if (threadIdx.x == 0 && qtile == 0 && h == 0) raise_flag(p.err_flag, PA_FLAG_LEN_OOB);
    return;
  }
  const int qr0 = qtile * kPfTile;                 // first query row of this CTA (within seq)
  if (qr0 >= q_len) return;
  const int cached = k_len - q_len;
  // keys needed by the CTA: up to the causal limit of its last row
  const int kv_end = min(k_len, cached + min(q_len, qr0 + kPfTile));
  const int ntiles = (kv_end + kPfTile - 1) / kPfTile;
  // rows of the last tile past the CTA's last visible key must be zeroed before
  // P V reads them (stale pool rows may hold NaN, rows no box filled hold
  // anything, and 0 * NaN = NaN); the producer warp does it and signals `ready`
  const int last_valid = kv_end - (ntiles - 1) * kPfTile;
  const bool zero_tail = last_valid < kPfTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kPfWarps);
    }
    mbar_init(ready, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kPfWarps) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks;
      const int box = p.box_rows;
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % STAGES;
        if (it >= STAGES && !pf_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, p.err_flag))
          break;
        const int t0 = it * kPfTile;
        const int tlen = min(kPfTile, kv_end - t0);
        const int nbox = (tlen + box - 1) / box;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox * box * 128 * HALVES * 2));
        uint8_t* kdst = smem + s * STAGE_BYTES;
        uint8_t* vdst = kdst + KV_BYTES;
        for (int b = 0; b < nbox; ++b) {
          const int t = t0 + b * box;
          const int bid = __ldg(bt + (t >> p.log2_bs));
          int row;
          if (bid < 0 || bid >= p.num_blocks) {
            raise_flag(p.err_flag, PA_FLAG_BLOCK_OOB);
            row = p.num_slots;
          } else {
            row = bid * p.block_size + (t & (p.block_size - 1));
          }
#pragma unroll
          for (int hf = 0; hf < HALVES; ++hf) {
            tma_load_3d(kdst + hf * HALF_BYTES + b * box * 128, &tmK, &full[s], hf * 64, kvh, row);
            tma_load_3d(vdst + hf * HALF_BYTES + b * box * 128, &tmV, &full[s], hf * 64, kvh, row);
          }
        }
      }
    }
    __syncwarp();
    if (zero_tail) {
      const int it = ntiles - 1;
      const int s = it % STAGES;
      if (pf_wait(&full[s], (it / STAGES) & 1, abort_flag, p.err_flag)) {
        uint8_t* vbase = smem + s * STAGE_BYTES + KV_BYTES;
        const int nrow = kPfTile - last_valid;
        for (int i = lane; i < nrow * 8 * HALVES; i += 32) {
          const int hf = i / (nrow * 8);
          const int rr = (i / 8) % nrow;
          *reinterpret_cast<uint4*>(vbase + hf * HALF_BYTES + (last_valid + rr) * 128 +
                                    (i & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(ready);
    }
    return;
  }

  const int r = lane >> 2, c = lane & 3;
  const int mi = lane >> 3, ri = lane & 7;
  const int wrow0 = qr0 + warp * 16;               // first query row of this warp (within seq)
  uint32_t qa[KSTEPS][4];
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = wrow0 + r + (j & 1) * 8;
      const int col = ks * 16 + c * 2 + (j >> 1) * 8;
      qa[ks][j] = row < q_len ? *reinterpret_cast<const uint32_t*>(
                                    p.q + (int64_t)(q_start + row) * p.q_stride + (int64_t)h * D + col)
                              : 0u;
    }
  // causal limits of this thread's two rows (absolute key positions)
  const int lim0 = cached + wrow0 + r;
  const int lim1 = lim0 + 8;

  float o[NT_O][4];
#pragma unroll
  for (int n = 0; n < NT_O; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  for (int it = 0; it < ntiles; ++it) {
    const int s = it % STAGES;
    if (!pf_wait(&full[s], (it / STAGES) & 1, abort_flag, p.err_flag)) break;
    uint8_t* kbase = smem + s * STAGE_BYTES;
    uint8_t* vbase = kbase + KV_BYTES;
    const int t0 = it * kPfTile;
    if (zero_tail && it == ntiles - 1 && !pf_wait(ready, 0, abort_flag, p.err_flag)) break;
    // warps whose rows all precede this tile skip it (their keys are all masked)
    if (t0 <= cached + wrow0 + 15) {
      float sc[NT_S][4];
#pragma unroll
      for (int n = 0; n < NT_S; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int hf = ks >> 2;
#pragma unroll
        for (int n2 = 0; n2 < NT_S / 2; ++n2) {
          const int tok = n2 * 16 + (mi >> 1) * 8 + ri;
          const int chunk = (ks & 3) * 2 + (mi & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(kbase + hf * HALF_BYTES) + sw128(tok, chunk), b0, b1, b2, b3);
          mma_bf16_16816(sc[2 * n2], qa[ks], b0, b1);
          mma_bf16_16816(sc[2 * n2 + 1], qa[ks], b2, b3);
        }
      }
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < NT_S; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = t0 + n * 8 + c * 2 + (e & 1);
          const int lim = (e >> 1) ? lim1 : lim0;
          const float v = (t <= lim && t < k_len) ? sc[n][e] * p.scale_log2 : -INFINITY;
          sc[n][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
      float alpha[2], rs[2] = {0.f, 0.f}, mref[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
        mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
        const float m_new = fmaxf(m_run[hh], mx[hh]);
        // a row with nothing visible yet keeps m = -inf; use 0 as its reference
        mref[hh] = m_new == -INFINITY ? 0.f : m_new;
        alpha[hh] = fast_exp2(m_run[hh] - mref[hh]);
        m_run[hh] = m_new;
      }
#pragma unroll
      for (int n = 0; n < NT_S; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pv = fast_exp2(sc[n][e] - mref[e >> 1]);
          sc[n][e] = pv;
          rs[e >> 1] += pv;
        }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) l_run[hh] = l_run[hh] * alpha[hh] + rs[hh];
#pragma unroll
      for (int n = 0; n < NT_O; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[1];
        o[n][3] *= alpha[1];
      }
#pragma unroll
      for (int kk = 0; kk < kPfTile / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
        pa[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
        pa[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
        pa[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
        for (int n2 = 0; n2 < D / 16; ++n2) {
          const int hf = (n2 * 16) >> 6;
          const int tok = kk * 16 + (mi & 1) * 8 + ri;
          const int chunk = ((n2 * 16) & 63) / 8 + (mi >> 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(vbase + hf * HALF_BYTES) + sw128(tok, chunk), b0, b1, b2, b3);
          mma_bf16_16816(o[2 * n2], pa, b0, b1);
          mma_bf16_16816(o[2 * n2 + 1], pa, b2, b3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 1);
    l_run[hh] += __shfl_xor_sync(0xffffffffu, l_run[hh], 2);
  }
  const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
  const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
  const int row0 = wrow0 + r, row1 = row0 + 8;
#pragma unroll
  for (int n = 0; n < NT_O; ++n) {
    const int col = n * 8 + c * 2;
    if (row0 < q_len)
      *reinterpret_cast<uint32_t*>(p.out + ((int64_t)(q_start + row0) * p.hq + h) * D + col) =
          pack_bf16(o[n][0] * inv0, o[n][1] * inv0);
    if (row1 < q_len)
      *reinterpret_cast<uint32_t*>(p.out + ((int64_t)(q_start + row1) * p.hq + h) * D + col) =
          pack_bf16(o[n][2] * inv1, o[n][3] * inv1);
  }
}

template <int D>
static pa_status launch_prefill_mma_d(const PrefillArgs& a, const CUtensorMap& mk,
                                      const CUtensorMap& mv, const PrefillMmaParams& prm) {
  constexpr int STAGE_BYTES = 2 * (D / 64) * kPfTile * 128;
  const size_t smem = (size_t)kPfStages * STAGE_BYTES + 1024 + (2 * kPfStages + 1) * 8 + 16;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(prefill_mma_kernel<D, kPfStages>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "prefill smem attribute");
    attr_done = true;
  }
  dim3 grid((a.max_seqlen_q + kPfTile - 1) / kPfTile, a.hq, a.num_seqs);
  cudaError_t e = launch_pdl(prefill_mma_kernel<D, kPfStages>, grid, dim3(kPfThreads), smem,
                             a.stream, mk, mv, prm);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return PA_OK;
}

pa_status launch_prefill_mma(const PrefillArgs& a) {
  const int box = a.block_size < kPfTile ? a.block_size : kPfTile;
  const int64_t slots = (int64_t)a.num_blocks * a.block_size;
  CUtensorMap mk, mv;
  pa_status s = get_tensor_map(&mk, a.k_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  s = get_tensor_map(&mv, a.v_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  PrefillMmaParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(a.q);
  prm.q_stride = a.q_stride;
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
  if (a.hq > 65535) return fail(PA_ERR_UNSUPPORTED, "too many heads");
  if (a.d == 128) return launch_prefill_mma_d<128>(a, mk, mv, prm);
  return launch_prefill_mma_d<64>(a, mk, mv, prm);
}

pa_status launch_prefill_tc(const PrefillArgs& a);

// head_dim 128 runs on the tcgen05 kernel; PA_PREFILL_PATH=mma selects the
// mma.sync kernel instead (both are GPU kernels; the switch exists to compare them).
pa_status launch_prefill(const PrefillArgs& a) {
  static const bool force_mma = [] {
    const char* e = getenv("PA_PREFILL_PATH");
    return e && strcmp(e, "mma") == 0;
  }();
  if (a.d == 128 && !force_mma) return launch_prefill_tc(a);
  return launch_prefill_mma(a);
}

}  // namespace pa
