// prefill_tc.cu -- varlen causal prefill over the paged pool on the 5th-gen
// tensor cores (tcgen05 + TMEM), head_dim 64 or 128.
//
// Definition: sequence i computes q_len new queries over k_len keys, the
// first k_len - q_len a cached prefix shared through the hash prefix cache
// ("Prefix Caching via hashing", lnwmold.com item); query j attends keys
// 0 .. k_len-q_len+j (bottom-right causal); prompts are batched by cumulative
// sequence lengths ("Preparation before computation", same item).  Query head
// h reads KV head h / G.
//
// Tiles.  The G query heads of one KV head share every K/V byte, so an MMA
// tile packs qpt = floor(128 / G) consecutive queries x the G heads of one KV
// head as its M rows (row r = query r / G, head r % G; G = 7: 18 queries x 7
// heads = 126 rows).  One TMA box {64 hdim, G heads, qpt queries} of the packed
// q lands exactly in that row order.  A tile's keys end at its last query's
// position, so the causal band wasted inside a tile is qpt keys wide instead
// of 128.
//
// Work unit = two consecutive query tiles (A = the later, B) of one
// (sequence, KV head), reading the same K/V tiles; its cost is the number of
// KV tiles tile A reads.  The kernel is persistent (one CTA per SM).  Units
// are listed from the most KV tiles to the fewest (bucket = tile A's KV tiles;
// within a bucket by sequence, pair, KV head) and dealt out in a snake: CTA c
// of G takes list positions c, 2G-1-c, 2G+c, 4G-1-c, ..., so the expensive
// units go first and every CTA ends close to the mean.  The producer warp
// walks this list (32 sequences per step, warp prefix sums; the bucket of a
// pair follows in closed form from the sequence's lengths) and hands each unit
// to the other roles through a 4-slot queue in shared memory.  The K/V
// ring streams across unit boundaries and the next unit's Q and first S
// overlap the current unit's epilogue.
//
// Roles (11 warps; 12 with the fused store):
//   warp 8   producer: stages the unit's block-table entries in shared memory
//            (one round trip), then Q tiles (one box per head-dim half) into
//            two Q buffers and 128-key K and V tiles (one box per
//            physical-block chunk, 128-byte swizzle) into a 5-slot ring.
//            With the fused store the new keys' boxes come from the step's
//            new-row arrays instead of the pool.
//   warps 9, 10   MMA issuers of tiles A and B (one thread each): S_t(j) =
//            Q_t K_j^T into the TMEM S columns (M=128, N=128, K=16 steps);
//            O_t += P_t(j) V_j with P read from TMEM (TS form, B = V MN-major);
//            per tile S_t(j+1) and P_t(j) V_j are issued in whichever order
//            their inputs become ready (the S columns' turn; P_t), so the
//            tensor core works on one tile while the other tile's softmax runs
//            and no P V waits behind the S columns.
//   warps 0-3 / 4-7   softmax of tile A / B, one thread per M row (TMEM lane):
//            causal mask on the tiles that reach past a row's last key; online
//            softmax in the log2 domain with a lazy rescale (the reference max
//            moves only when it grows by more than 8, i.e. 256x); exponentials
//            on the MUFU unit (a polynomial on the FMA pipe, Exp2Poly, can take
//            a share of them: kEmuPairs); P as bf16 pairs in the tile's TMEM
//            P columns; epilogue O / l -> bf16 -> global in 32-byte stores.
//            The warps of a tile that reads the unit's last V tile zero its rows
//            past the unit's last key (up to the next multiple of 16: P V skips
//            the 16-key steps beyond) before handing over P (stale pool rows may
//            hold NaN, and 0 * NaN = NaN in P V).
//   warp 11  (fused store only) writes the step's new K/V rows to their pool
//            slots: the tokens of each of the CTA's units, walking the unit
//            list on its own, since attention does not read those rows back.
// TMEM: 512 columns: S (128, shared by the tiles in turn) | P_A (64) | P_B (64) |
// O_A | O_B.  A tile's softmax releases the S columns as soon as S is in its
// registers, so the next Q K^T overlaps the exponentials instead of waiting
// for P V; P_t is rewritten only after the previous P_t V has completed, and a
// unit's first P V into O_t is issued only after tile t's softmax warps,
// which also run its epilogue, have read the previous unit's O_t.
// Every wait is bounded; an abort winds all roles down, drains the issued
// MMAs and frees TMEM.

#include <cmath>

#include "pa_common.cuh"
#include "pa_internal.h"
#include "tc_common.cuh"

namespace pa {

constexpr int kTcRows = 128;     // MMA M: packed (query, head) rows of a tile
constexpr int kTcKeys = 128;     // keys per KV tile (MMA N of QK^T, K of PV)
constexpr int kTcThreads = 352;  // 2 softmax warpgroups + producer warp + 2 MMA warps
// with the fused store, warp 11 writes the batch's new K/V rows to the pool;
// the register budget is that of 12 warps (3 per SM sub-partition) either way
constexpr int kTcBoundThreads = 384;
constexpr int kTcHalf = kTcRows * 128;  // one 128-row x 64-element bf16 half (swizzled)
constexpr int kRing = 5;         // K/V ring slots (K_j, V_j, K_j+1, ... in turn)
// TMEM columns: S (shared by the two tiles in turn), P_A, P_B (bf16 pairs), O_A, O_B
constexpr uint32_t kTmemS = 0, kTmemP = 128, kTmemO = 256;
constexpr float kLazyRescale = 8.f;   // log2 of the largest un-rescaled growth (256x)

// Exponentials evaluated by polynomial: pair k of every 8 value pairs (16
// scores) is emulated when bit k is set.
constexpr uint32_t kEmuPairs = 0x0;    // none: measured faster (the MUFU is not the limiter)

struct PrefillTcParams {
  __nv_bfloat16* out;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* block_tables;
  int max_blocks, num_seqs;
  int hq, hkv, group, qpt, rows;
  int block_size, log2_bs, box_rows;
  int num_blocks, num_slots;
  int max_seqlen_q, max_seqlen_k, total_q;
  int buckets;                     // KV tiles of the longest tile: ceil(max_seqlen_k / 128)
  float scale_log2;
  int32_t* err_flag;
  // fused store (slots != nullptr): new K/V rows [total_q, hkv, D] and their pool slots
  const int32_t* slots;
  const uint4* new_k;
  const uint4* new_v;
  int64_t new_k_stride16, new_v_stride16;   // 16-byte chunks between tokens
  uint4* kc;
  uint4* vc;
};

// One work unit: tiles A (t = 0) and B (t = 1) of a (sequence, KV head).
struct TcUnit {
  int seq, kvh, q_start, q_len, k_len, cached;
  int q0[2];        // first query of tile t within the sequence
  int nt[2];        // KV tiles tile t reads (nt[1] == 0: no tile B)
  int kv_end;       // keys tile A reads (tile B reads no more)
};

struct TcSeq {
  int q_start, q_len, k_len, T, P;   // T query tiles, P pairs
  bool ok;
};

__device__ __forceinline__ TcSeq tc_seq(const PrefillTcParams& p, int s) {
  TcSeq r;
  const int cq0 = __ldg(p.cu_q + s), cq1 = __ldg(p.cu_q + s + 1);
  const int ck0 = __ldg(p.cu_k + s), ck1 = __ldg(p.cu_k + s + 1);
  r.q_start = cq0;
  r.q_len = cq1 - cq0;
  r.k_len = ck1 - ck0;
  r.ok = cq0 >= 0 && r.q_len >= 0 && cq1 <= p.total_q && r.k_len >= r.q_len &&
         r.q_len <= p.max_seqlen_q && r.k_len <= p.max_seqlen_k &&
         r.k_len <= p.max_blocks * p.block_size;
  r.T = r.ok ? (r.q_len + p.qpt - 1) / p.qpt : 0;
  r.P = (r.T + 1) / 2;
  return r;
}

// First pair (0 = the sequence's last two tiles) whose tile A reads at most b
// KV tiles, or P when none does.  Pair pp's tile A ends at query
// min(q_len, (T - 2 pp) qpt), so it reads ceil((cached + that) / 128) KV
// tiles, which falls as pp grows.
__device__ __forceinline__ int tc_first_pair(const TcSeq& q, int b, int qpt) {
  const int cached = q.k_len - q.q_len;
  if (cached + q.q_len <= b * kTcKeys) return 0;
  const int R = b * kTcKeys - cached;
  if (R < 0) return q.P;
  return min(max((q.T - R / qpt + 1) / 2, 1), q.P);
}

// The unit list, walked by the producer warp (every lane calls find with the
// same, increasing positions; the results are warp-uniform).  The current
// window's per-sequence values stay in registers until the walk moves on.
struct TcWalk {
  int b;         // current bucket
  int s0;        // first sequence of the current window of 32
  int64_t base;  // list position of the window's first unit
  bool have;     // the lane values below belong to (b, s0)
  int cnt, lo, incl, total;   // this lane's sequence in the window: units, first pair, prefix
  int q_s0;      // the window whose lengths q holds (-1: none): with at most 32 sequences
                 // the lengths are read once, not once per bucket
  TcSeq q;
  __device__ __forceinline__ void init(const PrefillTcParams& p) {
    b = p.buckets;
    s0 = 0;
    base = 0;
    have = false;
    q_s0 = -1;
  }
  // Fills u with the unit at list position pos; false past the end.  With
  // `report`, invalid sequence lengths raise PA_FLAG_LEN_OOB (once per CTA).
  __device__ __forceinline__ bool find(const PrefillTcParams& p, int64_t pos, int lane, bool report,
                                       TcUnit& u) {
    while (b > 0) {
      if (!have) {
        const int s = s0 + lane;
        cnt = 0;
        lo = 0;
        if (q_s0 != s0) {
          q = s < p.num_seqs ? tc_seq(p, s) : TcSeq{};
          if (s < p.num_seqs && !q.ok && report && b == p.buckets)
            raise_flag(p.err_flag, PA_FLAG_LEN_OOB);
          q_s0 = s0;
        }
        if (s < p.num_seqs && q.P > 0) {
          lo = tc_first_pair(q, b, p.qpt);
          cnt = (tc_first_pair(q, b - 1, p.qpt) - lo) * p.hkv;
        }
        incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        total = __shfl_sync(0xffffffffu, incl, 31);
        have = true;
      }
      if (pos < base + total) {
        const int l = __ffs(__ballot_sync(0xffffffffu, base + incl > pos)) - 1;
        const int64_t first = base + __shfl_sync(0xffffffffu, incl - cnt, l);
        const int off = (int)(pos - first);
        const int pp = __shfl_sync(0xffffffffu, lo, l) + off / p.hkv;
        u.seq = s0 + l;
        u.kvh = off % p.hkv;
        u.q_start = __shfl_sync(0xffffffffu, q.q_start, l);
        u.q_len = __shfl_sync(0xffffffffu, q.q_len, l);
        u.k_len = __shfl_sync(0xffffffffu, q.k_len, l);
        const int T = __shfl_sync(0xffffffffu, q.T, l);
        u.cached = u.k_len - u.q_len;
        const int ta = T - 1 - 2 * pp, tb = ta - 1;
        u.q0[0] = ta * p.qpt;
        u.kv_end = u.cached + min(u.q_len, u.q0[0] + p.qpt);
        u.nt[0] = (u.kv_end + kTcKeys - 1) / kTcKeys;
        if (tb >= 0) {
          u.q0[1] = tb * p.qpt;
          u.nt[1] = (u.cached + min(u.q_len, u.q0[1] + p.qpt) + kTcKeys - 1) / kTcKeys;
        } else {
          u.q0[1] = 0;
          u.nt[1] = 0;
        }
        return true;
      }
      base += total;
      have = false;
      s0 += 32;
      if (s0 >= p.num_seqs) {
        s0 = 0;
        --b;
      }
    }
    return false;
  }
};

// List position of this CTA's k-th unit (snake order).
__device__ __forceinline__ int64_t tc_position(int k) {
  const int64_t g = gridDim.x;
  return (int64_t)(k >> 1) * 2 * g + ((k & 1) ? 2 * g - 1 - blockIdx.x : blockIdx.x);
}

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

// The same bounded wait as one inline-PTX loop, for waits taken while the
// softmax holds a full S row in registers (a C++ loop there makes the
// compiler spill the row): polls the phase, gives up when another role has
// aborted or after kWaitLimitNs.
__device__ __forceinline__ bool tc_wait_inline(uint64_t* bar, uint32_t parity,
                                               volatile int* abort_flag, int32_t* err_flag) {
  uint32_t res;
  asm volatile(
      "{\n\t"
      ".reg .pred P1;\n\t"
      ".reg .u64 T0, T1;\n\t"
      ".reg .u32 AB;\n\t"
      "mov.u64 T0, %%globaltimer;\n"
      "TCW_LOOP:\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
      "@P1 bra TCW_DONE;\n\t"
      "ld.volatile.shared.u32 AB, [%3];\n\t"
      "setp.ne.u32 P1, AB, 0;\n\t"
      "@P1 bra TCW_ABORT;\n\t"
      "mov.u64 T1, %%globaltimer;\n\t"
      "sub.u64 T1, T1, T0;\n\t"
      "setp.lt.u64 P1, T1, %4;\n\t"
      "@P1 bra TCW_LOOP;\n\t"
      "mov.u32 %0, 0;\n\t"
      "bra TCW_END;\n"
      "TCW_ABORT:\n\t"
      "mov.u32 %0, 2;\n\t"
      "bra TCW_END;\n"
      "TCW_DONE:\n\t"
      "mov.u32 %0, 1;\n"
      "TCW_END:\n\t"
      "}"
      : "=r"(res)
      : "r"(smem_u32(bar)), "r"(parity), "r"(smem_u32(const_cast<int*>(abort_flag))),
        "l"(kWaitLimitNs)
      : "memory");
  if (res == 0) {
    *abort_flag = 1;
    raise_flag(err_flag, PA_FLAG_TIMEOUT);
  }
  return res == 1;
}

// Waits until the shared counter reaches `target` (acquire), bounded like tc_wait.
__device__ __forceinline__ bool tc_wait_count(uint32_t* ctr, uint32_t target,
                                              volatile int* abort_flag, int32_t* err_flag) {
  const uint32_t a = smem_u32(ctr);
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    if ((int32_t)(v - target) >= 0) return true;
    if (i == 0) t0 = globaltimer_ns();
    if ((i & 255u) == 255u) {
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
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for two values on the FMA pipe.  x is clamped to >= -125 (2^-125 is
// below anything that survives the bf16 rounding of P next to a 1; below the
// clamp the result is exactly 0, as for masked scores), then
// split as x = j + f with j the nearest integer (adding and subtracting
// 1.5 * 2^23 rounds to an integer in the low mantissa bits) and f in
// [-0.5, 0.5]; 2^f is a cubic whose coefficients were fitted to minimise the
// relative error on that interval (iteratively reweighted least squares; max
// relative error 7.5e-5, against 2^-9 for the bf16 rounding of P), and j is
// added to the exponent field.
struct Exp2Poly {
  uint64_t magic, neg_magic, neg_one, c3, c2, c1, c0;
  __device__ __forceinline__ Exp2Poly() {
    magic = f32x2(12582912.f, 12582912.f);
    neg_magic = f32x2(-12582912.f, -12582912.f);
    neg_one = f32x2(-1.f, -1.f);
    c3 = f32x2(0.0551706925f, 0.0551706925f);
    c2 = f32x2(0.2426096499f, 0.2426096499f);
    c1 = f32x2(0.6932610273f, 0.6932610273f);
    c0 = f32x2(0.9999281764f, 0.9999281764f);
  }
  __device__ __forceinline__ void eval(float x0, float x1, float& e0, float& e1) const {
    const uint64_t x = f32x2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
    const uint64_t t = fadd2(x, magic);              // j + 1.5 * 2^23
    const uint64_t f = ffma2(fadd2(t, neg_magic), neg_one, x);   // x - j
    uint64_t q = ffma2(f, c3, c2);
    q = ffma2(q, f, c1);
    q = ffma2(q, f, c0);
    float q0, q1, t0, t1;
    f32x2_split(q, q0, q1);
    f32x2_split(t, t0, t1);
    e0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    e1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
    e0 = x0 > -125.f ? e0 : 0.f;                 // masked scores (-inf) give exactly 0
    e1 = x1 > -125.f ? e1 : 0.f;
  }
};

// Streaming 16-byte global accesses that leave L1 alone (the fused store
// touches each byte once).
__device__ __forceinline__ uint4 ld_stream16(const uint4* a) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(a));
  return v;
}
__device__ __forceinline__ void st_stream16(uint4* a, uint4 v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(a), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// One 32-byte global store (a full sector per lane): the epilogue's rows sit
// 256 bytes apart across a warp, so each store instruction touches 32 lines
// whatever its width, and 32-byte stores halve the instructions and the L1
// wavefronts of 16-byte ones.  `a` must be 32-byte aligned.
__device__ __forceinline__ void st_global32(void* a, uint4 lo, uint4 hi) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(a), "r"(lo.x),
               "r"(lo.y), "r"(lo.z), "r"(lo.w), "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
               : "memory");
}

// Fused store: copies the new K/V rows of a sequence's new tokens [r0, r1)
// (token r is key position cached + r) for KV head kvh to their pool slots.
// Per round of kRound tokens the warp reads the rows in 16-byte chunks spread
// over its lanes (kBatch loads in flight per lane) while lane j reads token
// j's slot (and, with `check`, its block-table slot: a slot that differs
// raises PA_FLAG_SLOT_MISMATCH, one past the pool PA_FLAG_SLOT_OOB), then
// writes the rows.  Negative and out-of-pool slots write nothing.
template <int D>
__device__ __forceinline__ void tc_store_rows(const PrefillTcParams& p, int q_start, int cached,
                                              const int32_t* bt, int kvh, int r0, int r1, int lane,
                                              bool check) {
  constexpr int C = D / 8;             // chunks of one K or V row
  constexpr int kPer = 2 * C;          // chunks of a token: K, then V
  constexpr int kTok = 32 / kPer;      // tokens one warp-wide access covers
  constexpr int kBatch = 16;           // accesses in flight per lane
  constexpr int kRound = kBatch * kTok;   // tokens per round (at most 32: one slot per lane)
  static_assert(kRound <= 32, "one slot per lane");
  const int c = lane % kPer, ch = c % C;
  const bool isv = c >= C;
  const uint4* src = (isv ? p.new_v : p.new_k) + kvh * C + ch;
  const int64_t sstride = isv ? p.new_v_stride16 : p.new_k_stride16;
  uint4* pool = (isv ? p.vc : p.kc) + kvh * C + ch;
  for (int g = r0; g < r1; g += kRound) {
    const int n = min(kRound, r1 - g);
    // the round's rows are read before, and independently of, their slots, so
    // the slot loads and the row loads are in flight together (one round trip)
    uint4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int t = u * kTok + lane / kPer;
      if (t < n) v[u] = ld_stream16(src + (int64_t)(q_start + g + t) * sstride);
    }
    int slot = -1;
    if (lane < n) {
      slot = __ldg(p.slots + q_start + g + lane);
      if (check) {
        const int k = cached + g + lane;
        const int bid = __ldg(bt + (k >> p.log2_bs));
        if (slot >= p.num_slots)
          raise_flag(p.err_flag, PA_FLAG_SLOT_OOB);
        else if (bid >= 0 && bid < p.num_blocks &&
                 slot != bid * p.block_size + (k & (p.block_size - 1)))
          raise_flag(p.err_flag, PA_FLAG_SLOT_MISMATCH);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int t = u * kTok + lane / kPer;
      const int sl = __shfl_sync(0xffffffffu, slot, t);
      if (t < n && sl >= 0 && sl < p.num_slots) st_stream16(pool + (int64_t)sl * p.hkv * C, v[u]);
    }
  }
}

constexpr int kBtCache = 256;    // block-table entries staged per unit
constexpr int kUnitSlots = 4;    // unit descriptors the producer publishes ahead
constexpr int kUnitReaders = 10; // the 2 MMA warps and the 8 softmax warps

struct TcBars {
  uint64_t q_full[2];      // Q tile t landed
  uint64_t q_empty[2];     // the last Q_t K^T of a unit is complete: Q buffer t free
  uint64_t kv_full[kRing];
  uint64_t kv_empty[kRing];
  uint64_t s_full[2];      // S_t is in the S columns
  // reads of tile t's S out of the S columns, counted per warp (4 per S): a
  // monotonic count, not an mbarrier phase, because an issuer may wait for
  // the other tile's next read before that tile's previous read is done,
  // which a parity wait would take for complete
  uint32_t s_reads[2];
  uint64_t p_full[2];      // P_t is in its TMEM columns (O_t rescaled if needed)
  uint64_t pv_done[2];     // the last P_t V issued is complete
  uint64_t drain[2];
  uint64_t unit_full[kUnitSlots];   // descriptor published (nt[0] == 0: no more units)
  uint64_t unit_empty[kUnitSlots];  // every reader has copied it
  TcUnit units[kUnitSlots];
  uint32_t tmem;
  int abort_flag;
  int bt[kBtCache];        // the producer's unit: its first block-table entries
};

// The k-th unit descriptor the producer published, read by a whole warp
// (warp-uniform result; false when the list is over or a wait gave up).
__device__ __forceinline__ bool tc_take_unit(TcBars* bar, uint32_t k, int lane,
                                             volatile int* abort_flag, int32_t* err_flag,
                                             TcUnit& u, bool& ok) {
  const uint32_t slot = k % kUnitSlots;
  bool got = true;
  if (lane == 0) got = tc_wait(&bar->unit_full[slot], (k / kUnitSlots) & 1, abort_flag, err_flag);
  if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
    ok = false;
    return false;
  }
  u = bar->units[slot];
  __syncwarp();
  if (lane == 0) mbar_arrive(&bar->unit_empty[slot]);
  return u.nt[0] > 0;
}

template <int D>
__global__ void __launch_bounds__(kTcBoundThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmNK,
                      const __grid_constant__ CUtensorMap tmNV, const PrefillTcParams p) {
  constexpr int kHalves = D / 64;
  constexpr uint32_t kOCols = D;               // TMEM columns of one O accumulator
  constexpr int kTile = kHalves * kTcHalf;     // one Q, K or V tile
  constexpr int kSteps = D / 16;               // K steps of Q K^T
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                     // [2 tiles]
  uint8_t* sKV = sQ + 2 * kTile;          // [kRing slots]
  TcBars* bar = reinterpret_cast<TcBars*>(sKV + kRing * kTile);
  volatile int* abort_flag = &bar->abort_flag;

  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 8 && lane == 0) {
    mbar_init(&bar->q_full[0], 1);
    mbar_init(&bar->q_full[1], 1);
    mbar_init(&bar->q_empty[0], 1);
    mbar_init(&bar->q_empty[1], 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&bar->kv_full[s], 1);
      mbar_init(&bar->kv_empty[s], 2);        // one commit per tile (both by A without B)
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar->s_full[t], 1);
      mbar_init(&bar->p_full[t], 4);
      mbar_init(&bar->pv_done[t], 1);
    }
    mbar_init(&bar->drain[0], 1);
    mbar_init(&bar->drain[1], 1);
    bar->s_reads[0] = 0;
    bar->s_reads[1] = 0;
    for (int s = 0; s < kUnitSlots; ++s) {
      mbar_init(&bar->unit_full[s], 1);
      mbar_init(&bar->unit_empty[s], kUnitReaders);
    }
    bar->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (p.slots) {
      tma_prefetch_desc(&tmNK);
      tma_prefetch_desc(&tmNV);
    }
  }
  // rows >= p.rows of the Q buffers are never written by TMA: zero them once so
  // the padding rows of S stay finite
  {
    const int pad = kTcRows - p.rows;
    for (int i = threadIdx.x; i < 2 * kHalves * pad * 8; i += blockDim.x) {
      const int chunk = i & 7, rr = (i >> 3) % pad, hb = (i >> 3) / pad;   // hb = buffer * kHalves + half
      *reinterpret_cast<uint4*>(sQ + hb * kTcHalf + (p.rows + rr) * 128 + chunk * 16) =
          make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 10) {
    tc::tmem_alloc(&bar->tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bar->tmem;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    uint32_t kv_i = 0, qn[2] = {0, 0};
    const int box = p.box_rows;
    TcWalk walk;
    walk.init(p);
    for (int k = 0;; ++k) {
      TcUnit u;
      const bool more = walk.find(p, tc_position(k), lane, true, u);
      if (!more) u.nt[0] = 0;                   // the end of this CTA's list
      // publish the unit to the MMA and softmax warps
      const uint32_t us = (uint32_t)k % kUnitSlots;
      bool free_slot = true;
      if (lane == 0 && k >= kUnitSlots)
        free_slot = tc_wait(&bar->unit_empty[us], ((k / kUnitSlots) - 1) & 1, abort_flag, p.err_flag);
      if (!__shfl_sync(0xffffffffu, free_slot ? 1 : 0, 0)) break;
      if (lane == 0) {
        bar->units[us] = u;
        mbar_arrive(&bar->unit_full[us]);
      }
      if (!more) break;
      const int n = u.nt[0];
      // the unit's block-table entries, staged in one round trip
      const int32_t* bt = p.block_tables + (int64_t)u.seq * p.max_blocks;
      const int nblk = min((u.kv_end + p.block_size - 1) >> p.log2_bs, kBtCache);
      for (int i = lane; i < nblk; i += 32) bar->bt[i] = __ldg(bt + i);
      // fused store: keys from the cached length on are read from the new-row
      // arrays, box by box; a box that holds both cached and new keys (cached
      // length not a multiple of the box) is read from the pool, so its new
      // rows are written there first (the store warp writes the same values)
      const bool fused = p.slots != nullptr;
      const int split = fused ? min(u.kv_end, (u.cached + box - 1) / box * box) : 0;
      if (fused && split > u.cached) {
        tc_store_rows<D>(p, u.q_start, u.cached, bt, u.kvh, 0, split - u.cached, lane, false);
        fence_proxy_async_global();
      }
      __syncwarp();
      bool ok = true;
      if (lane == 0) {
        for (int t = 0; t < 2 && ok; ++t) {
          if (u.nt[t] == 0) continue;
          if (qn[t] > 0 && !tc_wait(&bar->q_empty[t], (qn[t] - 1) & 1, abort_flag, p.err_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar->q_full[t], (uint32_t)(kHalves * p.rows * 128));
#pragma unroll
          for (int hf = 0; hf < kHalves; ++hf)
            tma_load_3d(sQ + t * kTile + hf * kTcHalf, &tmQ, &bar->q_full[t], hf * 64,
                        u.kvh * p.group, u.q_start + u.q0[t]);
          ++qn[t];
        }
        for (int j = 0; j < n && ok; ++j) {
          const int t0 = j * kTcKeys;
          const int nbox = (min(kTcKeys, u.kv_end - t0) + box - 1) / box;
          const uint32_t bytes = (uint32_t)(nbox * box * 128 * kHalves);
          int rows[kTcKeys / 16];
          for (int b = 0; b < nbox; ++b) {
            const int t = t0 + b * box;
            if (fused && t >= split) {                 // new keys: token rows of the arrays
              rows[b] = -1 - (u.q_start + t - u.cached);
              continue;
            }
            const int lb = t >> p.log2_bs;
            const int bid = lb < kBtCache ? bar->bt[lb] : __ldg(bt + lb);
            if (bid < 0 || bid >= p.num_blocks) {
              raise_flag(p.err_flag, PA_FLAG_BLOCK_OOB);
              rows[b] = p.num_slots;                 // past the pool: TMA fills zeros
            } else {
              rows[b] = bid * p.block_size + (t & (p.block_size - 1));
            }
          }
          for (int kv = 0; kv < 2; ++kv, ++kv_i) {
            const int slot = kv_i % kRing;
            if (kv_i >= kRing &&
                !tc_wait(&bar->kv_empty[slot], ((kv_i / kRing) - 1) & 1, abort_flag, p.err_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bar->kv_full[slot], bytes);
            for (int b = 0; b < nbox; ++b) {
              uint8_t* dst = sKV + slot * kTile + b * box * 128;
              const bool arr = rows[b] < 0;
              const CUtensorMap* map = arr ? (kv ? &tmNV : &tmNK) : (kv ? &tmV : &tmK);
              const int row = arr ? -1 - rows[b] : rows[b];
#pragma unroll
              for (int hf = 0; hf < kHalves; ++hf)
                tma_load_3d(dst + hf * kTcHalf, map, &bar->kv_full[slot], hf * 64, u.kvh, row);
            }
          }
        }
      }
      // lane 0 is done with this unit's staged block table before it is overwritten
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
    }
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 9 issues tile A's MMAs, warp 10 tile B's (lane 0; the warp takes
    // the unit descriptors).  Per tile, S_t(j+1) and P_t(j) V_j are issued in
    // whichever order their inputs become ready, so the tile's next S is
    // usually computed while its softmax runs and a P V never waits behind the
    // S columns.  The S columns are used in one fixed order, A0 B0 A1 B1 ...
    // (A alone once B has no more KV tiles), and every S waits until the
    // previous S in that order has been read into registers; each P V waits
    // only for its own tile's P.  (The protocol was checked by a model of all
    // roles and of the asynchronous copies and MMAs under random schedules: no
    // deadlock, no wait whose parity could alias another phase, and no
    // unordered conflicting access other than the two tiles' identical zero
    // writes to the last V tile.)
    const int t = warp - 9;
    constexpr uint32_t idS = tc::idesc_bf16(kTcRows, kTcKeys, false, false);
    constexpr uint32_t idO = tc::idesc_bf16(kTcRows, D, false, true);
    // descriptors are built once; stepping K adds (byte offset / 16) to the
    // start-address field (no carry: shared addresses stay below 256 KB)
    const uint64_t dQ = tc::sdesc_sw128(smem_u32(sQ + t * kTile), 16, 1024);
    const uint64_t dK0 = tc::sdesc_sw128(smem_u32(sKV), 16, 1024);
    const uint64_t dV0 = tc::sdesc_sw128(smem_u32(sKV), kTcHalf, 1024);
    uint32_t kv_i = 0, qc = 0, pc = 0;
    // S groups of each tile in earlier units, and the last S of the previous
    // unit (tile, index in that tile's sequence; tile -1: none yet)
    uint32_t ra = 0, rb = 0;
    int last_t = -1;
    uint32_t last_i = 0;
    auto wait_kv = [&](uint32_t i) {
      return tc_wait(&bar->kv_full[i % kRing], (i / kRing) & 1, abort_flag, p.err_flag);
    };
    // S_t(j) = Q_t K_j^T into the shared S columns, once the S before it in
    // the order (tile pt, pi-th S of that tile) has been read.
    auto issue_s = [&](int pt, uint32_t pi, uint32_t kslot) {
      if (pt >= 0 && !tc_wait_count(&bar->s_reads[pt], 4 * (pi + 1), abort_flag, p.err_flag))
        return false;
      tc::fence_after_sync();
      const uint64_t dK = dK0 + (uint64_t)((kslot * kTile) >> 4);
#pragma unroll
      for (int ks = 0; ks < kSteps; ++ks) {
        const uint64_t o = (uint64_t)(((ks >> 2) * kTcHalf + (ks & 3) * 32) >> 4);
        tc::mma_ss(tmem + kTmemS, dQ + o, dK + o, idS, ks > 0);
      }
      tc::commit(&bar->s_full[t]);
      return true;
    };
    for (uint32_t k = 0;; ++k) {
      TcUnit u;
      bool ok = true;
      if (!tc_take_unit(bar, k, lane, abort_flag, p.err_flag, u, ok)) break;
      const int n = u.nt[0], nb = u.nt[1], nt = u.nt[t];
      if (lane == 0 && nt > 0) {
        // the S read before S_t(j) in the order A0 B0 A1 B1 ... A(nb) ... A(n-1)
        auto pred_t = [&](int j) -> int {
          return t == 1 ? 0 : (j == 0 ? last_t : (j - 1 < nb ? 1 : 0));
        };
        auto pred_i = [&](int j) -> uint32_t {
          return t == 1 ? ra + j : (j == 0 ? last_i : (j - 1 < nb ? rb + j - 1 : ra + j - 1));
        };
        // K_j / V_j are released by one commit of each tile (tile A commits
        // twice for the tiles B does not read)
        auto release = [&](uint32_t slot, int j) {
          tc::commit(&bar->kv_empty[slot]);
          if (t == 0 && j >= nb) tc::commit(&bar->kv_empty[slot]);
        };
        ok = tc_wait(&bar->q_full[t], qc++ & 1, abort_flag, p.err_flag) && wait_kv(kv_i);
        if (ok) {
          tc::fence_after_sync();
          ok = issue_s(pred_t(0), pred_i(0), kv_i % kRing);
          if (ok) {
            if (nt == 1) tc::commit(&bar->q_empty[t]);
            release(kv_i % kRing, 0);                       // K_0
          }
        }
        for (int j = 0; ok && j < nt; ++j) {
          const uint32_t iv = kv_i + 2 * j + 1, vslot = iv % kRing;
          const uint32_t kn = iv + 1, kslot = kn % kRing;  // K_j+1
          // S_t(j+1) and P_t(j) V_j in whichever order their inputs become
          // ready: S_t(j+1) waits for the other tile's read of the S columns,
          // and a P V held behind that wait would hold up this tile's
          // softmax, which rewrites P_t only after P_t V has completed
          bool s_todo = j + 1 < nt, pv_todo = true;
          const int spt = s_todo ? pred_t(j + 1) : -1;
          const uint32_t spi = s_todo ? pred_i(j + 1) : 0;
          uint64_t w0 = 0;
          for (uint32_t spin = 0; s_todo || pv_todo; ++spin) {
            bool progressed = false;
            if (s_todo && mbar_test_wait(&bar->kv_full[kn % kRing], (kn / kRing) & 1)) {
              uint32_t v = 4 * (spi + 1);
              if (spt >= 0)
                asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];"
                             : "=r"(v) : "r"(smem_u32(&bar->s_reads[spt])) : "memory");
              if ((int32_t)(v - 4 * (spi + 1)) >= 0) {
                issue_s(-1, 0, kslot);                    // (its predecessor was read: no wait)
                if (j + 2 == nt) tc::commit(&bar->q_empty[t]);
                release(kslot, j + 1);
                s_todo = false;
                progressed = true;
              }
            }
            if (pv_todo && mbar_test_wait(&bar->kv_full[vslot], (iv / kRing) & 1) &&
                mbar_test_wait(&bar->p_full[t], pc & 1)) {
              ++pc;
              // O_t += P_t V_j (the last KV tile: only the 16-key steps before
              // kv_end; both tiles' softmax warps zero V rows past the last key
              // up to the next multiple of 16 before handing over P)
              tc::fence_after_sync();
              const uint64_t dV = dV0 + (uint64_t)((vslot * kTile) >> 4);
              const int nks = j == n - 1 ? (u.kv_end - j * kTcKeys + 15) / 16 : kTcKeys / 16;
#pragma unroll
              for (int ks = 0; ks < kTcKeys / 16; ++ks)
                if (ks < nks)
                  tc::mma_ts(tmem + kTmemO + kOCols * t, tmem + kTmemP + 64 * t + ks * 8,
                             dV + (uint64_t)((ks * 2048) >> 4), idO, (j > 0 || ks > 0));
              tc::commit(&bar->pv_done[t]);
              release(vslot, j);                            // V_j
              pv_todo = false;
              progressed = true;
            }
            if (!progressed && (spin & 255u) == 255u) {
              if (*abort_flag) {
                ok = false;
                break;
              }
              const uint64_t now = globaltimer_ns();
              if (w0 == 0) {
                w0 = now;
              } else if (now - w0 > kWaitLimitNs) {
                *abort_flag = 1;
                raise_flag(p.err_flag, PA_FLAG_TIMEOUT);
                ok = false;
                break;
              }
            }
          }
        }
      }
      if (nb == n) {
        last_t = 1;
        last_i = rb + nb - 1;
      } else {
        last_t = 0;
        last_i = ra + n - 1;
      }
      ra += n;
      rb += nb;
      kv_i += 2 * n;
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
    }
    if (lane == 0) {
      // every issued MMA finishes before TMEM is released
      tc::commit(&bar->drain[t]);
      mbar_wait(&bar->drain[t], 0);
    }
    __syncwarp();
  } else if (warp == 11) {
    // ------------------------------------------------------------ fused store
    // (present only with the fused store) each unit's own tokens, tile B's
    // first query to tile A's last, for the unit's KV head: every (token, KV
    // head) of the batch belongs to exactly one unit, so each new row is
    // written once.  Attention reads the new rows from the arrays, so nothing
    // waits for these writes: this warp walks the CTA's unit list on its own
    // and runs ahead of the other roles instead of taking the published units.
    TcWalk walk;
    walk.init(p);
    for (int k = 0;; ++k) {
      TcUnit u;
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;   // warp-uniform: the walk shuffles
      if (!walk.find(p, tc_position(k), lane, false, u)) break;
      const int r0 = u.nt[1] > 0 ? u.q0[1] : u.q0[0];
      const int r1 = min(u.q_len, u.q0[0] + p.qpt);
      tc_store_rows<D>(p, u.q_start, u.cached, p.block_tables + (int64_t)u.seq * p.max_blocks,
                       u.kvh, r0, r1, lane, true);
    }
  } else {
    // ------------------------------------------------------------ softmax (warpgroup t = tile)
    const int t = warp >> 2;                       // 0: tile A, 1: tile B
    const int r = threadIdx.x & 127;               // M row = TMEM lane
    const int qi = r / p.group, hh = r - qi * p.group;   // query within the tile, head in the group
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + kTmemS + lane_off;
    const uint32_t tP = tmem + kTmemP + 64 * t + lane_off;
    const uint32_t tO = tmem + kTmemO + kOCols * t + lane_off;
    const float sl2 = p.scale_log2;
    const Exp2Poly ex;
    uint32_t sc = 0, pvc = 0;
    uint32_t kv_i = 0;                             // ring index of the unit's K_0 (tile A tracks it)
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      TcUnit u;
      if (!tc_take_unit(bar, k, lane, abort_flag, p.err_flag, u, ok)) break;
      const uint32_t kv_unit = kv_i;
      kv_i += 2 * u.nt[0];
      if (u.nt[t] == 0) continue;
      const int nt = u.nt[t], q0 = u.q0[t];
      const int limit = min(u.cached + q0 + qi, u.k_len - 1);   // last visible key of this row
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < nt; ++j) {
        if (!__all_sync(0xffffffffu, tc_wait(&bar->s_full[t], sc++ & 1, abort_flag, p.err_flag))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        float sv[kTcKeys];
        tc::ld128(tS, reinterpret_cast<uint32_t*>(sv));
        tc::wait_ld();
        // S is in registers: the next Q K^T may overwrite the S columns
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          asm volatile("red.release.cta.shared::cta.add.u32 [%0], 1;" ::"r"(smem_u32(&bar->s_reads[t]))
                       : "memory");
        }
        const int t0 = j * kTcKeys;
        if (t0 + kTcKeys - 1 > limit) {            // tile reaches past the row's last key: mask
          const int lim = limit - t0;
#pragma unroll
          for (int i = 0; i < kTcKeys; ++i) sv[i] = i <= lim ? sv[i] : -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = fmaxf(sv[2 * c], sv[2 * c + 1]);
#pragma unroll
        for (int i = 16; i < kTcKeys; i += 16) {
#pragma unroll
          for (int c = 0; c < 8; ++c) mx8[c] = max3f(mx8[c], sv[i + 2 * c], sv[i + 2 * c + 1]);
        }
        const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7])) * sl2;  // scale > 0
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
        uint64_t rs2[4] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f), f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
        // P as 64 bf16 pairs (kept in registers until the previous P_t V is done)
        uint32_t pk[kTcKeys / 2];
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {
#pragma unroll
          for (int i = 64 * hk; i < 64 * hk + 64; i += 2) {
            float x0, x1, e0, e1;
            f32x2_split(ffma2(f32x2(sv[i], sv[i + 1]), sc2, nm2), x0, x1);
            if ((kEmuPairs >> ((i >> 1) & 7)) & 1) {
              ex.eval(x0, x1, e0, e1);
            } else {
              e0 = fast_exp2(x0);
              e1 = fast_exp2(x1);
            }
            rs2[(i >> 1) & 3] = fadd2(rs2[(i >> 1) & 3], f32x2(e0, e1));
            pk[i >> 1] = pack_bf16(e0, e1);
          }
        }
        // the previous P_t V must be complete before P_t is overwritten and O_t rescaled
        if (j > 0 && !__all_sync(0xffffffffu,
                                 tc_wait_inline(&bar->pv_done[t], pvc++ & 1, abort_flag, p.err_flag))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        tc::st64(tP, pk);
        if (j == u.nt[0] - 1) {
          // the unit's last V tile: P V reads its rows up to the next multiple of
          // 16 past the last key; zero those past the last key first (both
          // tiles' warps write the same zeros, each before its own P V)
          const int last_valid = u.kv_end - j * kTcKeys;
          if (last_valid & 15) {
            const uint32_t iv = kv_unit + 2 * j + 1, slot = iv % kRing;
            if (!__all_sync(0xffffffffu, tc_wait(&bar->kv_full[slot], (iv / kRing) & 1, abort_flag,
                                                 p.err_flag))) {
              ok = false;
              break;
            }
            const int nrow = 16 - (last_valid & 15);
            for (int i = r; i < nrow * 8 * kHalves; i += kTcRows) {
              const int hf = i / (nrow * 8);
              const int rr = (i >> 3) % nrow;
              *reinterpret_cast<uint4*>(sKV + slot * kTile + hf * kTcHalf + (last_valid + rr) * 128 +
                                        (i & 7) * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
        }
        {
          float a0, a1, b0, b1;
          f32x2_split(fadd2(rs2[0], rs2[2]), a0, a1);
          f32x2_split(fadd2(rs2[1], rs2[3]), b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
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
      if (!ok) break;
      // epilogue: O / l -> bf16
      if (!__all_sync(0xffffffffu, tc_wait(&bar->pv_done[t], pvc++ & 1, abort_flag, p.err_flag))) break;
      tc::fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool store = r < p.rows && q0 + qi < u.q_len;
      __nv_bfloat16* orow =
          p.out + ((int64_t)(u.q_start + q0 + qi) * p.hq + u.kvh * p.group + hh) * D;
      uint32_t ov[D];
      if (D == 128) {
        tc::ld128(tO, ov);
      } else {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tc::ld32(tO + c * 32, ov + c * 32);
      }
      tc::wait_ld();
      // O / l, two columns per packed multiply
      const uint64_t inv2 = f32x2(inv, inv);
#pragma unroll
      for (int m = 0; m < D / 2; ++m) {
        float a, b;
        f32x2_split(fmul2(f32x2(__uint_as_float(ov[2 * m]), __uint_as_float(ov[2 * m + 1])), inv2), a, b);
        ov[2 * m] = __float_as_uint(a);
        ov[2 * m + 1] = __float_as_uint(b);
      }
      // 8 output columns of this row as bf16
      auto pack8 = [&](int k) {
        uint4 v;
        v.x = pack_bf16(__uint_as_float(ov[8 * k + 0]), __uint_as_float(ov[8 * k + 1]));
        v.y = pack_bf16(__uint_as_float(ov[8 * k + 2]), __uint_as_float(ov[8 * k + 3]));
        v.z = pack_bf16(__uint_as_float(ov[8 * k + 4]), __uint_as_float(ov[8 * k + 5]));
        v.w = pack_bf16(__uint_as_float(ov[8 * k + 6]), __uint_as_float(ov[8 * k + 7]));
        return v;
      };
      if (store) {
        // rows are D * 2 bytes apart: 32-byte stores when the base allows
        if ((reinterpret_cast<uintptr_t>(p.out) & 31u) == 0) {
#pragma unroll
          for (int k = 0; k < D / 8; k += 2) st_global32(orow + k * 8, pack8(k), pack8(k + 1));
        } else {
#pragma unroll
          for (int k = 0; k < D / 8; ++k) *reinterpret_cast<uint4*>(orow + k * 8) = pack8(k);
        }
      }
      // the next unit's first P V overwrites O_t: every lane's reads are done
      tc::fence_before_sync();
      __syncwarp();
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 10) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int D>
static pa_status launch_prefill_d(const PrefillArgs& a) {
  constexpr int kTile = (D / 64) * kTcHalf;
  const int group = a.hq / a.hkv;
  if (group > kTcRows) return fail(PA_ERR_UNSUPPORTED, "prefill: more than 128 query heads per KV head");
  const int qpt = kTcRows / group;
  const int box = a.block_size < kTcKeys ? a.block_size : kTcKeys;
  const int64_t slots = (int64_t)a.num_blocks * a.block_size;
  CUtensorMap mq, mk, mv;
  pa_status s = get_tensor_map(&mq, a.q, a.total_q, a.hq, a.d, a.q_stride, qpt, group);
  if (s != PA_OK) return s;
  s = get_tensor_map(&mk, a.k_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  s = get_tensor_map(&mv, a.v_cache, slots, a.hkv, a.d, (int64_t)a.hkv * a.d, box);
  if (s != PA_OK) return s;
  const bool fused = a.slot_mapping != nullptr;
  CUtensorMap mnk = mk, mnv = mv;                // the new-row arrays (fused store only)
  if (fused) {
    s = get_tensor_map(&mnk, a.key, a.total_q, a.hkv, a.d, a.key_stride, box);
    if (s != PA_OK) return s;
    s = get_tensor_map(&mnv, a.value, a.total_q, a.hkv, a.d, a.value_stride, box);
    if (s != PA_OK) return s;
  }
  PrefillTcParams prm{};
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.cu_q = a.cu_q;
  prm.cu_k = a.cu_k;
  prm.block_tables = a.block_tables;
  prm.max_blocks = a.max_blocks;
  prm.num_seqs = a.num_seqs;
  prm.hq = a.hq;
  prm.hkv = a.hkv;
  prm.group = group;
  prm.qpt = qpt;
  prm.rows = qpt * group;
  prm.block_size = a.block_size;
  prm.log2_bs = __builtin_ctz((unsigned)a.block_size);
  prm.box_rows = box;
  prm.num_blocks = a.num_blocks;
  prm.num_slots = (int)slots;
  prm.max_seqlen_q = a.max_seqlen_q;
  prm.max_seqlen_k = a.max_seqlen_k;
  prm.total_q = a.total_q;
  prm.buckets = (a.max_seqlen_k + kTcKeys - 1) / kTcKeys;
  const int64_t max_pairs = ((int64_t)(a.max_seqlen_q + qpt - 1) / qpt + 1) / 2;
  const int64_t max_units = max_pairs * a.num_seqs * a.hkv;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.err_flag = a.err_flag;
  if (fused) {
    prm.slots = a.slot_mapping;
    prm.new_k = static_cast<const uint4*>(a.key);
    prm.new_v = static_cast<const uint4*>(a.value);
    prm.new_k_stride16 = a.key_stride / 8;
    prm.new_v_stride16 = a.value_stride / 8;
    prm.kc = static_cast<uint4*>(const_cast<void*>(a.k_cache));
    prm.vc = static_cast<uint4*>(const_cast<void*>(a.v_cache));
  }
  // at least 120 KB so that two CTAs never share an SM (each allocates all 512
  // TMEM columns)
  static_assert((2 + kRing) * (size_t)kTile + 1024 + sizeof(TcBars) <= 232448,
                "prefill shared memory exceeds the 227 KB a CTA may use");
  size_t smem = (2 + kRing) * (size_t)kTile + 1024 + sizeof(TcBars);
  if (smem < 120 * 1024) smem = 120 * 1024;
  s = ensure_smem_attr((const void*)prefill_tc_kernel<D>, (int)smem, "prefill smem attribute");
  if (s != PA_OK) return s;
  const int64_t ctas = max_units < device_sm_count() ? max_units : device_sm_count();
  cudaError_t e = launch_pdl(prefill_tc_kernel<D>, dim3((unsigned)ctas),
                             dim3(fused ? kTcThreads + 32 : kTcThreads), smem, a.stream, mq, mk,
                             mv, mnk, mnv, prm);
  if (e != cudaSuccess) {
    forget_smem_attr((const void*)prefill_tc_kernel<D>);
    return cuda_fail(e, "prefill launch");
  }
  return PA_OK;
}

pa_status launch_prefill(const PrefillArgs& a) {
  if (a.d == 128) return launch_prefill_d<128>(a);
  return launch_prefill_d<64>(a);
}

}  // namespace pa
