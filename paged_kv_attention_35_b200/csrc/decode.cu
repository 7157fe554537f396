// decode.cu -- paged decode attention (one query token per sequence), GQA.
//
// Definition (the pages defer the attention formula to their unpublished part
// 2; this is standard scaled-dot-product attention): for sequence i, query
// head h and KV head g = h / G,
//     out[i,h] = softmax_t(scale * q[i,h] . K_i[t,g]) V_i[t,g],  t < context_lens[i],
// with row t of K_i / V_i at pool row block_tables[i][t / bs] * bs + t % bs
// ("From Sequences to Blocks", "Control plane vs. data plane", lnwmold.com
// item; PagedAttention blocks, intelliparadigm.com section 3.2).
//
// Design (B200, HBM-bound: every K/V byte is read exactly once):
//  * grid (partition, kv_head x q_tile, sequence).  A CTA owns partition_size
//    consecutive positions of one sequence and one KV head, and *all* query
//    heads of that KV head's GQA group (up to 16 per q_tile), so each KV byte
//    crosses HBM once no matter how large the group is.
//  * one producer warp streams 64-token K and V tiles into a STAGES-deep ring
//    of shared-memory buffers with TMA (3-D tensor map over the pool,
//    128-byte swizzle, boxes of min(bs, 64) rows per physical block, L2
//    evict-first), signalling mbarriers with transaction counts.
//  * four consumer warps each take 16 tokens of every tile.  The group's
//    query heads are the 16 rows of an mma.sync m16n8k16 tile (bf16 in, fp32
//    accumulate): S = Q K^T over head_dim, online softmax in the log2 domain
//    with quad shuffles, O += P V.  Tensor cores here only keep the ALU off
//    the critical path (GQA 7 is 7 flop/byte, at the FP32-FMA ceiling); the
//    kernel stays bound by HBM.
//  * positions >= context_len in the last tile are masked to -inf and their V
//    rows zeroed in shared memory before P V (stale pool rows may hold NaN).
//  * fused store (pa_decode_store): in the CTA whose partition holds a
//    sequence's newest position, the consumer warp owning that position loads
//    the token's new K and V rows of its KV head at the start, writes them to
//    the pool at slot_mapping[seq] (the step's store_kvcache, for later steps)
//    and, once the last tile has landed in shared memory, overwrites the stale
//    row there -- no other CTA of the launch reads that slot, so no ordering
//    between the global store and the TMA reads is needed.
//  * the 4 warps merge (m, l, O) through shared memory; with one partition
//    the CTA writes bf16 output, otherwise fp32 partials for the reduce kernel.

#include <cmath>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kDecTile = 64;     // tokens per pipeline stage
constexpr int kDecWarps = 4;     // consumer warps, 16 tokens each
constexpr int kDecThreads = (kDecWarps + 1) * 32;
constexpr int kDecStages = 3;

struct DecodeParams {
  const __nv_bfloat16* q;
  int64_t q_stride;
  __nv_bfloat16* out;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  int hq, group, qtiles;
  int block_size, log2_bs, box_rows;
  int num_blocks, num_slots;
  float scale_log2;
  int partition, max_context_len, max_splits;
  float* ws_o;
  float* ws_ml;
  // fused store: null slots = plain decode
  const uint4* new_k;
  const uint4* new_v;
  int64_t new_k_stride16, new_v_stride16;   // 16-byte units between tokens
  const int32_t* slots;
  uint4* kc;
  uint4* vc;
  int hkv;
  int32_t* err_flag;
};

__device__ __forceinline__ int clamp_len(int L, const DecodeParams& p) {
  int cap = min(p.max_context_len, p.max_blocks * p.block_size);
  return L < 0 ? 0 : (L > cap ? cap : L);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
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

template <int D, int STAGES>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  constexpr int HALVES = D / 64;
  constexpr int HALF_BYTES = kDecTile * 128;       // 64 rows x 128 B
  constexpr int KV_BYTES = HALVES * HALF_BYTES;    // one K (or V) tile
  constexpr int STAGE_BYTES = 2 * KV_BYTES;
  constexpr int KSTEPS = D / 16;
  constexpr int NTILES_O = D / 8;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + STAGES);

  // No early griddepcontrol.launch_dependents here: the dependent merge
  // kernel's CTAs would become resident while this grid still has waves to
  // run, holding registers that a second decode CTA per SM needs (measured
  // 57.8 -> 56.5 us on the Qwen3-0.6B-shaped decode); it launches as this
  // grid's CTAs exit.
  pdl_wait();
  const int split = blockIdx.x;
  const int kvh = blockIdx.y / p.qtiles;
  const int qt = blockIdx.y % p.qtiles;
  const int seq = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int L_raw = __ldg(p.context_lens + seq);
  const int L = clamp_len(L_raw, p);
  if (threadIdx.x == 0 && split == 0 && blockIdx.y == 0 &&
      (L_raw <= 0 || L_raw > p.max_context_len || L_raw > p.max_blocks * p.block_size))
    raise_flag(p.err_flag, PA_FLAG_LEN_OOB);

  const int h0 = kvh * p.group + qt * 16;          // first query head of this CTA
  const int nh = min(16, p.group - qt * 16);       // query heads of this CTA
  const int t_begin = split * p.partition;

  if (L == 0) {                                    // empty sequence: zero output row
    if (split == 0)
      for (int i = threadIdx.x; i < nh * D; i += blockDim.x)
        p.out[((int64_t)seq * p.hq + h0 + i / D) * D + i % D] = __float2bfloat16(0.f);
    return;
  }
  if (t_begin >= L) return;
  const int t_end = min(L, t_begin + p.partition);
  const int ntiles = (t_end - t_begin + kDecTile - 1) / kDecTile;
  const int n_splits = (L + p.partition - 1) / p.partition;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kDecWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const uint64_t policy = policy_evict_first();
      const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks;
      const int box = p.box_rows;
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % STAGES;
        if (it >= STAGES &&
            !wait_or_abort(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, p.err_flag))
          break;
        const int tile_t0 = t_begin + it * kDecTile;
        const int tile_len = min(kDecTile, t_end - tile_t0);
        const int nbox = (tile_len + box - 1) / box;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(nbox * box * 128 * HALVES * 2));
        uint8_t* kdst = smem + s * STAGE_BYTES;
        uint8_t* vdst = kdst + KV_BYTES;
        for (int b = 0; b < nbox; ++b) {
          const int t = tile_t0 + b * box;
          const int bid = __ldg(bt + (t >> p.log2_bs));
          int row;
          if (bid < 0 || bid >= p.num_blocks) {
            raise_flag(p.err_flag, PA_FLAG_BLOCK_OOB);
            row = p.num_slots;                       // fully out of range: TMA fills zeros
          } else {
            row = bid * p.block_size + (t & (p.block_size - 1));
          }
#pragma unroll
          for (int hf = 0; hf < HALVES; ++hf) {
            tma_load_3d_hint(kdst + hf * HALF_BYTES + b * box * 128, &tmK, &full[s], hf * 64, kvh,
                             row, policy);
            tma_load_3d_hint(vdst + hf * HALF_BYTES + b * box * 128, &tmV, &full[s], hf * 64, kvh,
                             row, policy);
          }
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int r = lane >> 2;        // fragment row (query head within the tile) / 8-token column group
  const int c = lane & 3;
  // Q as A fragments: rows = query heads h0 + (0..15), k = head_dim
  uint32_t qa[KSTEPS][4];
  {
    const __nv_bfloat16* qrow = p.q + (int64_t)seq * p.q_stride + (int64_t)h0 * D;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = r + (j & 1) * 8;
        const int col = ks * 16 + c * 2 + (j >> 1) * 8;
        qa[ks][j] = row < nh ? *reinterpret_cast<const uint32_t*>(qrow + row * D + col) : 0u;
      }
    }
  }

  float o[NTILES_O][4];
#pragma unroll
  for (int n = 0; n < NTILES_O; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  const int tw = warp * 16;
  const int mi = lane >> 3, ri = lane & 7;

  // fused store: lanes 0..C-1 carry the K row's 16-byte chunks, C..2C-1 the V row's
  constexpr int C = D / 8;
  const int r_last = L - 1 - t_begin - (ntiles - 1) * kDecTile;   // newest position's tile row
  bool patch = false;                              // this lane patches the last tile
  uint4 nrow = make_uint4(0, 0, 0, 0);
  if (p.slots && t_end == L && r_last >= tw && r_last < tw + 16) {
    const int slot = __ldg(p.slots + seq);
    const int bid = __ldg(p.block_tables + (int64_t)seq * p.max_blocks + ((L - 1) >> p.log2_bs));
    const bool bid_ok = bid >= 0 && bid < p.num_blocks;
    const int expect = bid * p.block_size + ((L - 1) & (p.block_size - 1));
    const bool kv_lane = lane < 2 * C;
    const bool is_v = lane >= C;
    const int ch = lane % C;
    if (kv_lane)
      nrow = __ldg((is_v ? p.new_v + seq * p.new_v_stride16 : p.new_k + seq * p.new_k_stride16) +
                   kvh * C + ch);
    if (slot >= 0 && slot < p.num_slots) {
      // with a group of more than 16 query heads several CTAs (q tiles) share
      // this KV head: the first writes the pool row, every one patches its own
      // landed tile (no CTA of this launch reads the row back from the pool)
      if (kv_lane && qt == 0) (is_v ? p.vc : p.kc)[((int64_t)slot * p.hkv + kvh) * C + ch] = nrow;
      patch = kv_lane && bid_ok && slot == expect;
      if (lane == 0 && qt == 0 && bid_ok && slot != expect)
        raise_flag(p.err_flag, PA_FLAG_SLOT_MISMATCH);
    } else if (slot >= p.num_slots && lane == 0 && qt == 0) {
      raise_flag(p.err_flag, PA_FLAG_SLOT_OOB);
    }
  }

  for (int it = 0; it < ntiles; ++it) {
    const int s = it % STAGES;
    if (!wait_or_abort(&full[s], (it / STAGES) & 1, abort_flag, p.err_flag)) break;
    const int valid = min(16, t_end - (t_begin + it * kDecTile + tw));
    uint8_t* kbase = smem + s * STAGE_BYTES;
    uint8_t* vbase = kbase + KV_BYTES;
    if (patch && it == ntiles - 1) {
      // the newest token's rows replace what the pool held at its position
      const int ch = lane % C;
      *reinterpret_cast<uint4*>((lane >= C ? vbase : kbase) + (ch >> 3) * HALF_BYTES +
                                sw128(r_last, ch & 7)) = nrow;
      fence_proxy_async_smem();                    // (the stage is not refilled: last tile)
    }
    __syncwarp();
    if (valid > 0) {
      if (valid < 16) {
        // zero V rows past the context (stale rows may be NaN; 0 * NaN = NaN)
        const int nrow = 16 - valid;
        for (int i = lane; i < nrow * 8 * HALVES; i += 32) {
          const int hf = i / (nrow * 8);
          const int rr = (i / 8) % nrow;
          const int ch = i & 7;
          *reinterpret_cast<uint4*>(vbase + hf * HALF_BYTES + (tw + valid + rr) * 128 + ch * 16) =
              make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // S = Q K^T (16 heads x 16 tokens)
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int hf = ks >> 2;
        const int tok = tw + (mi >> 1) * 8 + ri;
        const int chunk = (ks & 3) * 2 + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(kbase + hf * HALF_BYTES) + sw128(tok, chunk), b0, b1, b2, b3);
        mma_bf16_16816(sc[0], qa[ks], b0, b1);
        mma_bf16_16816(sc[1], qa[ks], b2, b3);
      }
      // scale (log2 domain) and mask positions past the context
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = n * 8 + c * 2 + (e & 1);
          const float v = col < valid ? sc[n][e] * p.scale_log2 : -INFINITY;
          sc[n][e] = v;
          mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
      }
      float alpha[2], rs[2] = {0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float m_new = fmaxf(m_run[h], mx[h]);   // finite: column 0 is valid
        alpha[h] = fast_exp2(m_run[h] - m_new);
        m_run[h] = m_new;
      }
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pv = fast_exp2(sc[n][e] - m_run[e >> 1]);
          sc[n][e] = pv;
          rs[e >> 1] += pv;
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) l_run[h] = l_run[h] * alpha[h] + rs[h];
#pragma unroll
      for (int n = 0; n < NTILES_O; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[1];
        o[n][3] *= alpha[1];
      }
      uint32_t pa[4];
      pa[0] = pack_bf16(sc[0][0], sc[0][1]);
      pa[1] = pack_bf16(sc[0][2], sc[0][3]);
      pa[2] = pack_bf16(sc[1][0], sc[1][1]);
      pa[3] = pack_bf16(sc[1][2], sc[1][3]);
      // O += P V
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        const int hf = (n2 * 16) >> 6;
        const int tok = tw + (mi & 1) * 8 + ri;
        const int chunk = ((n2 * 16) & 63) / 8 + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(vbase + hf * HALF_BYTES) + sw128(tok, chunk), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * n2], pa, b0, b1);
        mma_bf16_16816(o[2 * n2 + 1], pa, b2, b3);
      }
      if (valid < 16) fence_proxy_async_smem();   // zeroing precedes the next TMA write
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // row sums across the quad
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
  }

  // ----------------------------------------------------- merge the 4 warps
  named_bar_sync(1, kDecWarps * 32);       // every consumer is done with the ring
  constexpr int OS = D + 4;                // padded row stride (floats)
  float* ms = reinterpret_cast<float*>(smem);
  float* ls = ms + kDecWarps * 16;
  float* os = ls + kDecWarps * 16;         // [warp][16][OS]
  if (c == 0) {
    ms[warp * 16 + r] = m_run[0];
    ms[warp * 16 + r + 8] = m_run[1];
    ls[warp * 16 + r] = l_run[0];
    ls[warp * 16 + r + 8] = l_run[1];
  }
#pragma unroll
  for (int n = 0; n < NTILES_O; ++n) {
    const int col = n * 8 + c * 2;
    float* o0 = os + (warp * 16 + r) * OS + col;
    float* o1 = os + (warp * 16 + r + 8) * OS + col;
    o0[0] = o[n][0];
    o0[1] = o[n][1];
    o1[0] = o[n][2];
    o1[1] = o[n][3];
  }
  named_bar_sync(1, kDecWarps * 32);

  for (int i = threadIdx.x; i < nh * D; i += kDecWarps * 32) {
    const int row = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, ms[w * 16 + row]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float mw = ms[w * 16 + row];
      const float f = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
      acc += f * os[(w * 16 + row) * OS + d];
      lsum += f * ls[w * 16 + row];
    }
    const int h = h0 + row;
    if (n_splits == 1) {
      p.out[((int64_t)seq * p.hq + h) * D + d] = __float2bfloat16(acc / lsum);
    } else {
      const int64_t slot = ((int64_t)seq * p.hq + h) * p.max_splits + split;
      p.ws_o[slot * D + d] = acc;
      if (d == 0) {
        p.ws_ml[slot * 2] = M;
        p.ws_ml[slot * 2 + 1] = lsum;
      }
    }
  }
}

// Merge the partitions of each (sequence, query head): the global max M, then
// out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
template <int D>
__global__ void __launch_bounds__(D) decode_reduce_kernel(const DecodeParams p) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.x, seq = blockIdx.y, d = threadIdx.x;
  const int L = clamp_len(__ldg(p.context_lens + seq), p);
  const int n = (L + p.partition - 1) / p.partition;
  if (n <= 1) return;
  const int64_t base = ((int64_t)seq * p.hq + h) * p.max_splits;
  // eight partitions per round, all their loads issued before any use (the
  // kernel is latency-bound), merged online into (M, acc, lsum)
  float M = -INFINITY, acc = 0.f, lsum = 0.f;
  for (int s0 = 0; s0 < n; s0 += 8) {
    float mv[8], lv[8], ov[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool v = s0 + k < n;
      const int64_t sl = base + s0 + k;
      mv[k] = v ? __ldcg(p.ws_ml + sl * 2) : -INFINITY;
      lv[k] = v ? __ldcg(p.ws_ml + sl * 2 + 1) : 0.f;
      ov[k] = v ? __ldcg(p.ws_o + sl * D + d) : 0.f;
    }
    float Mn = M;
#pragma unroll
    for (int k = 0; k < 8; ++k) Mn = fmaxf(Mn, mv[k]);
    const float a = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
    acc *= a;
    lsum *= a;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float f = mv[k] == -INFINITY ? 0.f : fast_exp2(mv[k] - Mn);
      acc += f * ov[k];
      lsum += f * lv[k];
    }
    M = Mn;
  }
  p.out[((int64_t)seq * p.hq + h) * D + d] = __float2bfloat16(acc / lsum);
}

template <int D>
static pa_status launch_decode_d(const DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv,
                                 const DecodeParams& prm) {
  constexpr int HALVES = D / 64;
  constexpr int STAGE_BYTES = 2 * HALVES * kDecTile * 128;
  const size_t smem = (size_t)kDecStages * STAGE_BYTES + 1024 + 2 * kDecStages * 8 + 16;
  pa_status s = ensure_smem_attr((const void*)decode_kernel<D, kDecStages>, (int)smem,
                                 "decode smem attribute");
  if (s != PA_OK) return s;
  dim3 grid(a.max_splits, a.hkv * prm.qtiles, a.num_seqs);
  cudaError_t e = launch_pdl(decode_kernel<D, kDecStages>, grid, dim3(kDecThreads), smem, a.stream,
                             mk, mv, prm);
  if (e != cudaSuccess) {
    forget_smem_attr((const void*)decode_kernel<D, kDecStages>);
    return cuda_fail(e, "decode launch");
  }
  if (a.max_splits > 1) {
    e = launch_pdl(decode_reduce_kernel<D>, dim3(a.hq, a.num_seqs), dim3(D), 0, a.stream, prm);
    if (e != cudaSuccess) return cuda_fail(e, "decode reduce launch");
  }
  return PA_OK;
}

pa_status launch_decode(const DecodeArgs& a) {
  const int box = a.block_size < kDecTile ? a.block_size : kDecTile;
  const int64_t slots = (int64_t)a.num_blocks * a.block_size;
  CUtensorMap mk, mv;
  pa_status s = get_tensor_map(&mk, a.k_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  s = get_tensor_map(&mv, a.v_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  DecodeParams prm{};
  prm.q = static_cast<const __nv_bfloat16*>(a.q);
  prm.q_stride = a.q_stride;
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.block_tables = a.block_tables;
  prm.max_blocks = a.max_blocks;
  prm.context_lens = a.context_lens;
  prm.hq = a.hq;
  prm.group = a.hq / a.hkv;
  prm.qtiles = (prm.group + 15) / 16;
  prm.block_size = a.block_size;
  prm.log2_bs = __builtin_ctz((unsigned)a.block_size);
  prm.box_rows = box;
  prm.num_blocks = a.num_blocks;
  prm.num_slots = (int)slots;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.partition = a.partition;
  prm.max_context_len = a.max_context_len;
  prm.max_splits = a.max_splits;
  prm.ws_o = a.ws_o;
  prm.ws_ml = a.ws_ml;
  prm.slots = a.slots;
  if (a.slots) {
    prm.new_k = static_cast<const uint4*>(a.new_k);
    prm.new_v = static_cast<const uint4*>(a.new_v);
    prm.new_k_stride16 = a.new_k_stride / 8;
    prm.new_v_stride16 = a.new_v_stride / 8;
    prm.kc = static_cast<uint4*>(const_cast<void*>(a.k_cache));
    prm.vc = static_cast<uint4*>(const_cast<void*>(a.v_cache));
  }
  prm.hkv = a.hkv;
  prm.err_flag = a.err_flag;
  if ((int64_t)a.hkv * prm.qtiles > 65535) return fail(PA_ERR_UNSUPPORTED, "too many heads");
  if (a.d == 128) return launch_decode_d<128>(a, mk, mv, prm);
  return launch_decode_d<64>(a, mk, mv, prm);
}

}  // namespace pa
