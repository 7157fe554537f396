// prefill_tc.cu -- varlen causal prefill over the paged pool on the 5th-gen
// tensor cores (tcgen05 + TMEM), head_dim 128.
//
// Definition (same as prefill_mma.cu): sequence i computes q_len new queries
// over k_len keys, the first k_len - q_len a cached prefix shared through the
// hash prefix cache ("Prefix Caching via hashing", lnwmold.com item); query j
// attends keys 0 .. k_len-q_len+j; prompts are batched by cumulative sequence
// lengths ("Preparation before computation", same item).
//
// One CTA = two consecutive 128-row query tiles (A, B) of one (sequence,
// query head); 10 warps:
//   warp 8      TMA producer: both Q tiles once, then 128-key K and V tiles of
//               the sequence (one box per physical-block chunk, 128-byte
//               swizzle) into a 5-slot ring (K_j, V_j, K_j+1, ...) shared by
//               both tiles; zeroes V rows of the last tile past the CTA's last
//               visible key (stale pool rows may hold NaN).
//   warp 9      MMA issuer (one thread): S_t(j) = Q_t K_j^T into tile t's TMEM
//               S buffer (M=128, N=128, K=16 x 8) and O_t += P_t(j) V_j into its
//               TMEM O accumulator (A = P read from TMEM, B = V MN-major),
//               interleaving the tiles so one tile's softmax overlaps the other
//               tile's MMAs; tcgen05.commit signals the mbarriers.
//   warps 0-3 / 4-7   softmax of tile A / B, one thread per query row (TMEM
//               lane): tcgen05.ld the S row, causal mask on diagonal tiles only,
//               online softmax in the log2 domain with a lazy rescale (the
//               reference max moves only when it grows by more than 8, a factor
//               256), P as bf16 pairs written back over the S columns it came
//               from (tcgen05.st), O rescaled in TMEM when needed; epilogue
//               O / l -> bf16 -> global.
// TMEM: 512 columns (S_A/P_A | O_A | S_B/P_B | O_B).  The MMA thread issues
// P V of a tile before that tile's next Q K^T, and tcgen05 MMAs of one thread
// run in issue order, so the next S never overwrites P before P V has read it.
// Shared memory: Q 2 x 32 KB, K/V ring 5 x 32 KB.  Every wait is bounded; an
// abort winds all roles down, drains the issued MMAs and frees TMEM.

#include <cmath>

#include "pa_common.cuh"
#include "pa_internal.h"
#include "tc_common.cuh"

namespace pa {

constexpr int kTcRows = 128;     // query rows per tile (MMA M)
constexpr int kTcKeys = 128;     // keys per KV tile (MMA N of QK^T, K of PV)
constexpr int kTcThreads = 320;  // 2 softmax warpgroups + producer warp + MMA warp
constexpr int kTile = 32768;     // one 128 x 128 bf16 operand: two 128 x 64 swizzled halves
constexpr int kHalf = 16384;
constexpr int kRing = 5;         // K/V ring slots (K_j, V_j, K_j+1, ... in turn)
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

// Packed / 3-input fp32 arithmetic of sm_100 (halves the softmax's issue slots).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

constexpr int kBtCache = 256;    // block-table entries staged in shared memory

// Barrier block in shared memory (after the operand buffers).
struct TcBars {
  uint64_t q_full;
  uint64_t kv_full[kRing];
  uint64_t kv_empty[kRing];
  uint64_t s_full[2];      // per query tile (A, B)
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t vz_ready;
  uint64_t drain;
  uint32_t tmem;
  int abort_flag;
  int bt[kBtCache];        // the sequence's first block-table entries
};

// One CTA = two consecutive 128-row query tiles (A, B) of one (sequence, head).
// The MMA thread interleaves them so that the softmax of one tile overlaps the
// other tile's P V and next Q K^T on the tensor core:
//   S_A(0) S_B(0) | PV_A(0) S_A(1) | PV_B(0) S_B(1) | PV_A(1) S_A(2) | ...
// Both tiles read the same K/V tiles (the later tile needs at most one more).
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const PrefillTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                     // [2 tiles]
  uint8_t* sKV = sQ + 2 * kTile;          // [kRing slots]
  TcBars* bar = reinterpret_cast<TcBars*>(sKV + kRing * kTile);
  volatile int* abort_flag = &bar->abort_flag;

  // pair 0 = the sequence's last two query tiles (they see the most keys), so
  // launch order is longest first and every CTA but possibly a sequence's
  // first carries two tiles; tile A is the later one of the pair.
  pdl_wait();
  pdl_trigger();
  const int pp = blockIdx.x;
  const int h = blockIdx.y, seq = blockIdx.z;
  const int kvh = h / p.group;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int cq0 = __ldg(p.cu_q + seq), cq1 = __ldg(p.cu_q + seq + 1);
  const int ck0 = __ldg(p.cu_k + seq), ck1 = __ldg(p.cu_k + seq + 1);
  const int q_start = cq0, q_len = cq1 - cq0, k_len = ck1 - ck0;
  if (!(cq0 >= 0 && q_len >= 0 && cq1 <= p.total_q && k_len >= q_len &&
        q_len <= p.max_seqlen_q && k_len <= p.max_seqlen_k && k_len <= p.max_blocks * p.block_size)) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && h == 0) raise_flag(p.err_flag, PA_FLAG_LEN_OOB);
    return;
  }
  const int T = (q_len + kTcRows - 1) / kTcRows;   // query tiles of the sequence
  if (2 * pp >= T) return;
  const int tile_a = T - 1 - 2 * pp, tile_b = tile_a - 1;
  const bool hasB = tile_b >= 0;
  const int q0A = tile_a * kTcRows;
  const int q0B = hasB ? tile_b * kTcRows : 0;
  const int cached = k_len - q_len;
  const int kv_endA = min(k_len, cached + min(q_len, q0A + kTcRows));
  const int kv_endB = hasB ? min(k_len, cached + min(q_len, q0B + kTcRows)) : 0;
  const int nA = (kv_endA + kTcKeys - 1) / kTcKeys;
  const int nB = (kv_endB + kTcKeys - 1) / kTcKeys;
  const int kv_end = max(kv_endA, kv_endB);
  const int n = max(nA, nB);
  const int last_valid = kv_end - (n - 1) * kTcKeys;
  const bool zero_tail = last_valid < kTcKeys;
  const int32_t* bt = p.block_tables + (int64_t)seq * p.max_blocks;

  if (warp == 8 && lane == 0) {
    // the producer thread sets up the barriers and starts the Q loads at once
    mbar_init(&bar->q_full, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&bar->kv_full[s], 1);
      mbar_init(&bar->kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar->s_full[t], 1);
      mbar_init(&bar->p_full[t], 4);
      mbar_init(&bar->pv_done[t], 1);
    }
    mbar_init(&bar->vz_ready, 1);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    mbar_arrive_expect_tx(&bar->q_full, hasB ? 2 * kTile : kTile);
    tma_load_3d(sQ, &tmQ, &bar->q_full, 0, h, q_start + q0A);
    tma_load_3d(sQ + kHalf, &tmQ, &bar->q_full, 64, h, q_start + q0A);
    if (hasB) {
      tma_load_3d(sQ + kTile, &tmQ, &bar->q_full, 0, h, q_start + q0B);
      tma_load_3d(sQ + kTile + kHalf, &tmQ, &bar->q_full, 64, h, q_start + q0B);
    }
  }
  if (warp == 8) {
    // stage the block-table entries this CTA reads (all lanes, one round trip)
    const int nblk = min((kv_end + p.block_size - 1) >> p.log2_bs, kBtCache);
    for (int i = lane; i < nblk; i += 32) bar->bt[i] = __ldg(bt + i);
  }
  if (warp == 9) {
    tc::tmem_alloc(&bar->tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // tile t: S at TMEM columns [256t, 256t+128) with P (bf16 pairs) over its first
  // 64 columns once S has been read; O at [256t+128, 256t+256)
  const uint32_t tmem = bar->tmem;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int box = p.box_rows;
      int i = 0;
      for (int j = 0; j < n; ++j) {
        const int t0 = j * kTcKeys;
        const int nbox = (min(kTcKeys, kv_end - t0) + box - 1) / box;
        const uint32_t bytes = (uint32_t)(nbox * box * 128 * 2);
        int rows[kTcKeys / 16];
        for (int b = 0; b < nbox; ++b) {
          const int t = t0 + b * box;
          const int lb = t >> p.log2_bs;
          const int bid = lb < kBtCache ? bar->bt[lb] : __ldg(bt + lb);
          if (bid < 0 || bid >= p.num_blocks) {
            raise_flag(p.err_flag, PA_FLAG_BLOCK_OOB);
            rows[b] = p.num_slots;                 // past the pool: TMA fills zeros
          } else {
            rows[b] = bid * p.block_size + (t & (p.block_size - 1));
          }
        }
        bool ok = true;
        for (int kv = 0; kv < 2; ++kv, ++i) {
          const int slot = i % kRing;
          if (i >= kRing &&
              !tc_wait(&bar->kv_empty[slot], ((i / kRing) - 1) & 1, abort_flag, p.err_flag)) {
            ok = false;
            break;
          }
          const CUtensorMap* map = kv ? &tmV : &tmK;
          mbar_arrive_expect_tx(&bar->kv_full[slot], bytes);
          for (int b = 0; b < nbox; ++b) {
            uint8_t* dst = sKV + slot * kTile + b * box * 128;
            tma_load_3d(dst, map, &bar->kv_full[slot], 0, kvh, rows[b]);
            tma_load_3d(dst + kHalf, map, &bar->kv_full[slot], 64, kvh, rows[b]);
          }
        }
        if (!ok) break;
      }
    }
    __syncwarp();
    if (zero_tail) {
      const int iv = 2 * (n - 1) + 1, slot = iv % kRing;
      if (tc_wait(&bar->kv_full[slot], (iv / kRing) & 1, abort_flag, p.err_flag)) {
        const int nrow = kTcKeys - last_valid;
        for (int t = lane; t < nrow * 16; t += 32) {
          const int hf = t / (nrow * 8);
          const int rr = (t / 8) % nrow;
          *reinterpret_cast<uint4*>(sKV + slot * kTile + hf * kHalf + (last_valid + rr) * 128 +
                                    (t & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->vz_ready);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(kTcRows, kTcKeys, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(kTcRows, 128, false, true);
      const int ntile[2] = {nA, nB};
      // descriptors are built once; stepping K adds (byte offset / 16) to the
      // start-address field (no carry: shared addresses stay below 256 KB)
      const uint64_t dQ0 = tc::sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = tc::sdesc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV0 = tc::sdesc_sw128(smem_u32(sKV), kHalf, 1024);
      auto issue_s = [&](int t, int j) {          // S_t(j) = Q_t K_j^T
        const int slot = (2 * j) % kRing;
        const uint64_t dQ = dQ0 + (uint64_t)((t * kTile) >> 4);
        const uint64_t dK = dK0 + (uint64_t)((slot * kTile) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t o = (uint64_t)(((ks >> 2) * kHalf + (ks & 3) * 32) >> 4);
          tc::mma_ss(tmem + 256 * t, dQ + o, dK + o, idS, ks > 0);
        }
        tc::commit(&bar->s_full[t]);
      };
      auto wait_k = [&](int j) {
        const int i = 2 * j;
        return tc_wait(&bar->kv_full[i % kRing], (i / kRing) & 1, abort_flag, p.err_flag);
      };
      bool ok = tc_wait(&bar->q_full, 0, abort_flag, p.err_flag) && wait_k(0);
      if (ok) {
        tc::fence_after_sync();
        issue_s(0, 0);
        if (nB > 0) issue_s(1, 0);
        tc::commit(&bar->kv_empty[0]);          // K_0 consumed by both tiles
      }
      for (int j = 0; ok && j < n; ++j) {
        const int iv = 2 * j + 1, vslot = iv % kRing;
        const bool vz = zero_tail && j == n - 1;
        // operands first (normally resident long before the softmax is done), so
        // nothing but the P handshake sits between consecutive MMA groups
        if (!tc_wait(vz ? &bar->vz_ready : &bar->kv_full[vslot], vz ? 0u : (uint32_t)((iv / kRing) & 1),
                     abort_flag, p.err_flag) ||
            (j + 1 < n && !wait_k(j + 1))) {
          ok = false;
          break;
        }
        for (int t = 0; t < 2; ++t) {
          if (j >= ntile[t]) continue;
          if (!tc_wait(&bar->p_full[t], j & 1, abort_flag, p.err_flag)) { ok = false; break; }
          tc::fence_after_sync();
          const uint64_t dV = dV0 + (uint64_t)((vslot * kTile) >> 4);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_ts(tmem + 256 * t + 128, tmem + 256 * t + ks * 8,
                       dV + (uint64_t)((ks * 2048) >> 4), idO, (j > 0 || ks > 0));
          if (j == ntile[t] - 1) tc::commit(&bar->pv_done[t]);   // the epilogue waits on it
          if (j + 1 < ntile[t]) issue_s(t, j + 1);
        }
        if (!ok) break;
        tc::commit(&bar->kv_empty[vslot]);                 // V_j consumed
        if (j + 1 < n) tc::commit(&bar->kv_empty[(2 * (j + 1)) % kRing]);   // K_j+1 consumed
      }
      // every issued MMA finishes before TMEM is released
      tc::commit(&bar->drain);
      mbar_wait(&bar->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (warpgroup t = tile)
    const int t = warp >> 2;                       // 0: tile A, 1: tile B
    const int r = threadIdx.x & 127;               // row within the tile = TMEM lane
    const int nt = t ? nB : nA;
    const int q0 = t ? q0B : q0A;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 256 * t + lane_off, tO = tS + 128;
    const int limit = min(cached + q0 + r, k_len - 1);   // last visible key of this row
    const float sl2 = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    float sv[kTcKeys];
    for (int j = 0; j < nt; ++j) {
      // S_t(j) complete implies every earlier MMA of this CTA -- P V of tile j-1
      // included -- is complete: O may be rescaled and the S/P columns reused.
      if (!tc_wait(&bar->s_full[t], j & 1, abort_flag, p.err_flag)) { ok = false; break; }
      tc::fence_after_sync();
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::ld32(tS + c * 32, reinterpret_cast<uint32_t*>(sv) + c * 32);
      tc::wait_ld();
      const int t0 = j * kTcKeys;
      if (t0 + kTcKeys - 1 > limit) {              // diagonal / tail tile: mask
        const int lim = limit - t0;
#pragma unroll
        for (int i = 0; i < kTcKeys; ++i) sv[i] = i <= lim ? sv[i] : -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int i = 0; i < kTcKeys; i += 8) {
        mx4[0] = max3f(mx4[0], sv[i + 0], sv[i + 1]);
        mx4[1] = max3f(mx4[1], sv[i + 2], sv[i + 3]);
        mx4[2] = max3f(mx4[2], sv[i + 4], sv[i + 5]);
        mx4[3] = max3f(mx4[3], sv[i + 6], sv[i + 7]);
      }
      const float mx = max3f(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2;  // scale > 0
      float alpha = 1.f;
      bool resc = false;
      if (m_ref == -INFINITY) {
        m_ref = mx;
      } else if (mx > m_ref + kLazyRescale) {
        alpha = fast_exp2(m_ref - mx);
        m_ref = mx;
        resc = true;
        l *= alpha;
      }
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
      const uint64_t sc2 = f32x2(sl2, sl2), nm2 = f32x2(neg_m, neg_m);
      uint64_t rs2[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
      uint32_t pk[kTcKeys / 2];
#pragma unroll
      for (int i = 0; i < kTcKeys; i += 2) {
        float x0, x1;
        f32x2_split(ffma2(f32x2(sv[i], sv[i + 1]), sc2, nm2), x0, x1);
        const float e0 = fast_exp2(x0), e1 = fast_exp2(x1);
        rs2[(i >> 1) & 1] = fadd2(rs2[(i >> 1) & 1], f32x2(e0, e1));
        pk[i >> 1] = pack_bf16(e0, e1);
      }
      {
        float a0, a1, b0, b1;
        f32x2_split(rs2[0], a0, a1);
        f32x2_split(rs2[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      tc::st32(tS, pk);                            // P over the first 64 S columns
      tc::st32(tS + 32, pk + 32);
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tc::ld32(tO + c * 32, ov);
          tc::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tc::st32(tO + c * 32, ov);
        }
      }
      tc::wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->p_full[t]);
    }
    // epilogue: O / l -> bf16
    if (nt > 0 && ok && tc_wait(&bar->pv_done[t], 0, abort_flag, p.err_flag)) {
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool store = q0 + r < q_len;
      __nv_bfloat16* orow = p.out + ((int64_t)(q_start + q0 + r) * p.hq + h) * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tc::ld32(tO + c * 32, ov);
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
  if (warp == 9) {
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
  const size_t smem = (2 + kRing) * (size_t)kTile + 1024 + sizeof(TcBars);
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "prefill_tc smem attribute");
    attr_done = true;
  }
  if (a.hq > 65535) return fail(PA_ERR_UNSUPPORTED, "too many heads");
  dim3 grid((a.max_seqlen_q + 2 * kTcRows - 1) / (2 * kTcRows), a.hq, a.num_seqs);
  cudaError_t e = launch_pdl(prefill_tc_kernel, grid, dim3(kTcThreads), smem, a.stream, mq, mk, mv,
                             prm);
  if (e != cudaSuccess) return cuda_fail(e, "prefill_tc launch");
  return PA_OK;
}

}  // namespace pa
