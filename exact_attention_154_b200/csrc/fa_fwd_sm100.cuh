// fa_fwd_sm100.cuh -- exact attention forward, O = softmax(scale * Q K^T [+ causal]) V,
// for Blackwell (sm_100a), with the per-row logsumexp.
//
// The method is the tiled online-softmax recurrence of flash_attention_forward
// in "flash_attention.py" (forceinjection.github.io): per query row a running
// max m, a running sum l and an unnormalised output O are updated once per
// key/value block and O / l is written at the end, so the N x N score matrix
// never leaves the SM.  The pages give that recurrence for 64 x 64 blocks on
// an NPU; what follows is a B200 design of the same arithmetic:
//
//   * one persistent CTA per SM walks a static list of work tiles
//     (b, h, 256 query rows = two 128-row Q tiles, or one for head dim 256);
//   * a TMA producer warp loads the Q tiles once per work tile and streams
//     128-row K and V tiles through a ring of shared-memory stages guarded by
//     full / empty mbarriers (128-byte swizzle, no cluster multicast);
//   * one thread of the MMA warp issues tcgen05 MMAs: S = Q K^T from shared
//     memory into tensor memory (TMEM), and O += P V with P read from TMEM and
//     V from shared memory, committing each group to an mbarrier;
//   * each softmax warpgroup owns one Q tile: thread t of the group owns query
//     row t (TMEM lane t), so row max and row sum need no shuffles.  It reads
//     S from TMEM, applies scale (in the log2 domain), the causal / ragged
//     mask, the online update, writes P as 16-bit pairs back over S in TMEM,
//     rescales O in TMEM when its reference max moved, and finally writes
//     O / l and the logsumexp.
//
// The running max used as the exp2 reference is only moved when the block max
// exceeds it by more than 2^8 (in log2 units 8): O, l and the reference stay
// mutually consistent, so the final O / l and LSE = ln2 * (m_ref + log2 l) are
// exact, and P stays below 256 -- well inside fp16 / bf16 range.
//
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel records
// a code in a device word, drains what it issued, frees TMEM and returns.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "sm100_ptx.cuh"

namespace fa_sm100 {

constexpr int BM = 128;  // query rows per Q tile (tcgen05 M)
constexpr int BN = 128;  // key / value rows per K or V tile
constexpr float kLazyRescaleLog2 = 8.0f;
// Argument pairs (of every 8) whose exp2 runs on the FMA pipe instead of MUFU.
#ifndef FA_POLY_PAIRS_PER8
#define FA_POLY_PAIRS_PER8 2
#endif
constexpr int kPolyPairsPer8 = FA_POLY_PAIRS_PER8;

// Error word written by a kernel whose bounded wait ran out: 0 = none,
// otherwise (role << 8) | site, first writer wins.
__device__ unsigned int g_fa_watchdog = 0u;

enum WaitSite : unsigned {
  kSiteQEmpty = 1, kSiteKvEmpty, kSiteQFull, kSiteKvFull, kSitePFull, kSiteSFull, kSiteODone,
  kSiteSelfTest, kSiteDrain
};
enum Role : unsigned { kRoleProducer = 1, kRoleMma = 2, kRoleSoftmax = 3, kRoleTest = 4 };

struct FwdParams {
  CUtensorMap tmap_q;  // 4-D (d, N, H, B) views of q, k, v, box (64, 128, 1, 1)
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  void* o;
  float* lse;  // [B, H, N] or nullptr
  long long o_stride_b, o_stride_h, o_stride_n;  // in elements
  int B, H, N;
  int causal;
  float scale_log2;  // scale * log2(e)
  int num_qblocks;   // query blocks per (b, h)
  int num_tiles;     // B * H * num_qblocks
  unsigned long long wait_limit_ns;
};

// Bounded wait on an mbarrier phase.  Gives up when the CTA-wide abort flag
// is raised or after `limit_ns`; the first to give up records `code`.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned long long limit_ns, unsigned code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicCAS(&g_fa_watchdog, 0u, code);
      return false;
    }
  }
}

template <int HD, int QS, int KVS, bool BF16>
struct FwdCfg {
  static_assert(HD == 64 || HD == 128 || HD == 256, "head dim");
  static_assert(QS == 1 || QS == 2, "Q tiles per work tile");
  static constexpr int CHUNKS = HD / 64;          // 128-byte column chunks per row
  static constexpr int CHUNK_BYTES = 128 * 128;   // one chunk of a 128-row tile
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;
  static constexpr int SOFTMAX_WARPS = 4 * QS;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;
  static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
  // whole warpgroups: the softmax groups, then one group holding the producer
  // warp, the MMA warp and two idle warps
  static constexpr int THREADS = 128 * (QS + 1);

  static constexpr int SQ_OFF = 0;
  static constexpr int SKV_OFF = QS * TILE_BYTES;
  static constexpr int BAR_OFF = SKV_OFF + KVS * TILE_BYTES;
  // barrier indices
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1, B_KV_FULL = 2, B_KV_EMPTY = 2 + KVS,
                       B_S_FULL = 2 + 2 * KVS, B_P_FULL = B_S_FULL + 2, B_O_DONE = B_P_FULL + 4,
                       B_DRAIN = B_O_DONE + 2, NUM_BARS = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack for 1024-B alignment
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");

  // TMEM columns (fp32 words): two S buffers, then the O accumulators.
  static constexpr uint32_t TMEM_COLS = 512;
  __host__ __device__ static constexpr uint32_t s_col(int buf) { return buf ? 128u : 0u; }
  static constexpr uint32_t O_COL0 = 256u;
  static constexpr uint32_t O_COL1 = 256u + HD;
  static_assert(256 + QS * HD <= 512, "TMEM budget");
};

struct TileInfo {
  int b, h, q0, diag0, n[2], n_max;
};

template <int QS>
__device__ __forceinline__ TileInfo decode_tile(const FwdParams& p, int t) {
  TileInfo ti;
  const int bh = t / p.num_qblocks;
  const int qi = t - bh * p.num_qblocks;
  // heaviest query blocks first within a head when causal
  const int qblock = p.causal ? (p.num_qblocks - 1 - qi) : qi;
  ti.b = bh / p.H;
  ti.h = bh - ti.b * p.H;
  ti.q0 = qblock * BM * QS;
  ti.diag0 = ti.q0 / BN;
  const int nkv = (p.N + BN - 1) / BN;
  ti.n_max = 0;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    int n = 0;
    if (s < QS && ti.q0 + s * BM < p.N) n = p.causal ? min(nkv, ti.diag0 + s + 1) : nkv;
    ti.n[s] = n;
    ti.n_max = max(ti.n_max, n);
  }
  return ti;
}

// Static persistent schedule: round r hands tiles [r*G, (r+1)*G) to the G
// CTAs, reversing the order on odd rounds so causal work evens out.
__device__ __forceinline__ int tile_of(int round, int cta, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ roles
template <int HD, int QS, int KVS, bool BF16>
__device__ void producer_role(const FwdParams& p, uint32_t base, volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, BF16>;
  const uint32_t bars = base + C::BAR_OFF;
  const int G = gridDim.x, cta = blockIdx.x;
  int kv_count = 0, q_count = 0;
  bool ok = true;
  for (int round = 0; ok && round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    if (q_count > 0) {
      ok = wait_phase(bars + 8 * C::B_Q_EMPTY, (q_count - 1) & 1, abort_flag, p.wait_limit_ns,
                      (kRoleProducer << 8) | kSiteQEmpty);
      if (!ok) break;
    }
    mbar_arrive_expect_tx(bars + 8 * C::B_Q_FULL, QS * C::TILE_BYTES);
#pragma unroll
    for (int s = 0; s < QS; ++s)
#pragma unroll
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_load_4d(base + C::SQ_OFF + s * C::TILE_BYTES + c * C::CHUNK_BYTES, &p.tmap_q,
                    bars + 8 * C::B_Q_FULL, c * 64, ti.q0 + s * BM, ti.h, ti.b);
    ++q_count;
    for (int j = 0; ok && j < ti.n_max; ++j) {
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const int slot = kv_count % KVS, use = kv_count / KVS;
        if (use > 0) {
          ok = wait_phase(bars + 8 * (C::B_KV_EMPTY + slot), (use - 1) & 1, abort_flag,
                          p.wait_limit_ns, (kRoleProducer << 8) | kSiteKvEmpty);
          if (!ok) break;
        }
        const uint32_t full = bars + 8 * (C::B_KV_FULL + slot);
        mbar_arrive_expect_tx(full, C::TILE_BYTES);
        const CUtensorMap* map = kv ? &p.tmap_v : &p.tmap_k;
#pragma unroll
        for (int c = 0; c < C::CHUNKS; ++c)
          tma_load_4d(base + C::SKV_OFF + slot * C::TILE_BYTES + c * C::CHUNK_BYTES, map, full,
                      c * 64, j * BN, ti.h, ti.b);
        ++kv_count;
      }
    }
  }
  if (!ok) {
    // Let the loads already issued land before the CTA's shared memory goes away.
    const unsigned long long drain = 10000000ull;
    volatile int no_abort_q = 0;
    if (q_count > 0)
      wait_phase(bars + 8 * C::B_Q_FULL, (q_count - 1) & 1, &no_abort_q, drain,
                 (kRoleProducer << 8) | kSiteDrain);
    for (int i = max(0, kv_count - KVS); i < kv_count; ++i) {
      volatile int no_abort = 0;
      const uint32_t bar = bars + 8 * (C::B_KV_FULL + i % KVS);
      if (!mbar_try_wait(bar, (i / KVS) & 1))
        wait_phase(bar, (i / KVS) & 1, &no_abort, drain, (kRoleProducer << 8) | kSiteDrain);
    }
  }
}

template <int HD, int QS, int KVS, bool BF16>
__device__ void mma_role(const FwdParams& p, uint32_t base, uint32_t tmem,
                         volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, BF16>;
  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t idesc_qk = f16_idesc(BF16, BM, BN, false);
  const uint32_t idesc_pv = f16_idesc(BF16, BM, HD, true);
  const unsigned long long lim = p.wait_limit_ns;
  const int G = gridDim.x, cta = blockIdx.x;
  int kv_count = 0, q_count = 0;
  uint32_t p_par[2] = {0u, 0u};
  int s_iter = 0, pv_iter = 0;  // single-Q-tile variant: S buffer ring position
  bool ok = true;

  auto wait_kv = [&](int idx) -> bool {
    const bool r = wait_phase(bars + 8 * (C::B_KV_FULL + idx % KVS), (idx / KVS) & 1, abort_flag,
                              lim, (kRoleMma << 8) | kSiteKvFull);
    tc_fence_after_sync();
    return r;
  };
  auto issue_s = [&](int s, uint32_t s_col, int kslot) {
    const uint32_t qa = base + C::SQ_OFF + s * C::TILE_BYTES;
    const uint32_t kb = base + C::SKV_OFF + kslot * C::TILE_BYTES;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t off = (kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32;
      mma_ss(tmem + s_col, sw128_desc(qa + off, 16, 1024), sw128_desc(kb + off, 16, 1024),
             idesc_qk, kk > 0 ? 1u : 0u);
    }
  };
  // O (+)= P V, P handed over in two halves of 64 keys: the first four K-steps
  // start as soon as the softmax has written the first half.
  auto issue_pv = [&](int bar, uint32_t o_col, uint32_t p_col, int vslot, bool accumulate) -> bool {
    const uint32_t vb = base + C::SKV_OFF + vslot * C::TILE_BYTES;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (!wait_phase(bars + 8 * (C::B_P_FULL + 2 * bar + half), p_par[bar], abort_flag, lim,
                      (kRoleMma << 8) | kSitePFull))
        return false;
      tc_fence_after_sync();
#pragma unroll
      for (int k4 = 0; k4 < BN / 32; ++k4) {
        const int kk = half * (BN / 32) + k4;
        mma_ts(tmem + o_col, tmem + p_col + kk * 8,
               sw128_desc(vb + kk * 16 * 128, C::CHUNK_BYTES, 1024), idesc_pv,
               (accumulate || kk > 0) ? 1u : 0u);
      }
    }
    p_par[bar] ^= 1u;
    return true;
  };

  for (int round = 0; ok && round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    ok = wait_phase(bars + 8 * C::B_Q_FULL, q_count & 1, abort_flag, lim,
                    (kRoleMma << 8) | kSiteQFull);
    tc_fence_after_sync();
    ++q_count;
    if (!ok) break;
    const int kv0 = kv_count;
    for (int j = 0; ok && j <= ti.n_max; ++j) {
      const int k_idx = kv0 + 2 * j, v_idx = kv0 + 2 * j - 1;
      if constexpr (QS == 2) {
        // order: PV0(j-1), S0(j), PV1(j-1), S1(j)
        if (j >= 1 && !(ok = wait_kv(v_idx))) break;
        bool k_ready = false;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const uint32_t o_col = s ? C::O_COL1 : C::O_COL0;
          if (j >= 1 && j <= ti.n[s]) {
            if (!(ok = issue_pv(s, o_col, C::s_col(s), v_idx % KVS, j > 1))) break;
            tc_commit(bars + 8 * (C::B_O_DONE + s));
          }
          if (j < ti.n[s]) {
            if (!k_ready) {
              if (!(ok = wait_kv(k_idx))) break;
              k_ready = true;
            }
            issue_s(s, C::s_col(s), k_idx % KVS);
            tc_commit(bars + 8 * (C::B_S_FULL + s));
          }
        }
        if (!ok) break;
        if (j < ti.n_max) tc_commit(bars + 8 * (C::B_KV_EMPTY + k_idx % KVS));
        if (j >= 1) tc_commit(bars + 8 * (C::B_KV_EMPTY + v_idx % KVS));
        if (j == ti.n_max - 1) tc_commit(bars + 8 * C::B_Q_EMPTY);
      } else {
        // order: S(j) into the other S buffer, then PV(j-1)
        if (j < ti.n_max) {
          if (!(ok = wait_kv(k_idx))) break;
          const int buf = s_iter & 1;
          issue_s(0, C::s_col(buf), k_idx % KVS);
          tc_commit(bars + 8 * (C::B_S_FULL + buf));
          tc_commit(bars + 8 * (C::B_KV_EMPTY + k_idx % KVS));
          if (j == ti.n_max - 1) tc_commit(bars + 8 * C::B_Q_EMPTY);
          ++s_iter;
        }
        if (j >= 1) {
          if (!(ok = wait_kv(v_idx))) break;
          if (!(ok = issue_pv(0, C::O_COL0, C::s_col(pv_iter & 1), v_idx % KVS, j > 1))) break;
          tc_commit(bars + 8 * C::B_O_DONE);
          tc_commit(bars + 8 * (C::B_KV_EMPTY + v_idx % KVS));
          ++pv_iter;
        }
      }
    }
    kv_count = kv0 + 2 * ti.n_max;
  }
  if (!ok) {
    // Wait for every MMA this thread issued before TMEM is released.
    volatile int no_abort = 0;
    tc_commit(bars + 8 * C::B_DRAIN);
    wait_phase(bars + 8 * C::B_DRAIN, 0, &no_abort, 10000000ull, (kRoleMma << 8) | kSiteDrain);
  }
}

// 2^x for two arguments on the FMA pipe: x = n + f with n = rint(x) taken from
// the low mantissa bits of x + 1.5 * 2^23, f in [-1/2, 1/2]; 2^f by a degree-3
// polynomial whose coefficients are the relative-error minimax fit on
// [-1/2, 1/2] (Remez exchange, max relative error 7.5e-5, below half an ulp of
// bf16 and fp16 P); 2^n applied by adding n to the exponent field.  Arguments
// are clamped at -126 so the exponent cannot wrap (2^-126 is ~0 here).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.9999280571937561f, c1 = 0.6932609677314758f,
                  c2 = 0.2426111251115799f, c3 = 0.0551716685295105f;
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
  const float2 n = __fadd2_rn(t, make_float2(-kRound, -kRound));
  const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
  float2 q = __ffma2_rn(make_float2(c3, c3), f, make_float2(c2, c2));
  q = __ffma2_rn(q, f, make_float2(c1, c1));
  q = __ffma2_rn(q, f, make_float2(c0, c0));
  float2 r;
  r.x = __int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23));
  r.y = __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23));
  return r;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Exponentials, row-sum and 16-bit packing of 32 consecutive scores.
// POLY8 of every 8 argument pairs go through exp2_poly2, the rest through ex2.
template <bool BF16, int POLY8>
__device__ __forceinline__ void softmax_chunk(const float* sv, float sl2, float neg_ref,
                                              uint32_t* pk, float2& acc) {
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const float2 x = __ffma2_rn(make_float2(sv[2 * q], sv[2 * q + 1]), make_float2(sl2, sl2),
                               make_float2(neg_ref, neg_ref));
    float2 e;
    if ((q % 8) >= 8 - POLY8) {
      e = exp2_poly2(x);
    } else {
      e.x = ex2(x.x);
      e.y = ex2(x.y);
    }
    acc = __fadd2_rn(acc, e);
    pk[q] = pack2<BF16>(e.x, e.y);
  }
}

template <int HD, int QS, int KVS, bool BF16>
__device__ void softmax_role(const FwdParams& p, uint32_t base, uint32_t tmem,
                             volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, BF16>;
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  const uint32_t bars = base + C::BAR_OFF;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int s = warp / 4;                   // which Q tile of the work tile
  const int r = (warp % 4) * 32 + lane;     // query row within the tile == TMEM lane
  const uint32_t lane_base = tmem + ((static_cast<uint32_t>(warp % 4) * 32u) << 16);
  const uint32_t o_col = s ? C::O_COL1 : C::O_COL0;
  const int bar_idx = (QS == 2) ? s : 0;
  const unsigned long long lim = p.wait_limit_ns;
  const float sl2 = p.scale_log2;
  const int G = gridDim.x, cta = blockIdx.x;
  uint32_t s_par[2] = {0u, 0u}, o_par = 0u;
  int s_iter = 0;

  for (int round = 0; round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    const int n = ti.n[s];
    if (n == 0) continue;
    const int row = ti.q0 + s * BM + r;
    // keys visible from this row: [0, limit)
    const int limit = p.causal ? min(row + 1, p.N) : p.N;
    float m_ref = -INFINITY, l = 0.f;

    for (int j = 0; j < n; ++j) {
      const int buf = (QS == 2) ? s : (s_iter & 1);
      const uint32_t s_col = C::s_col(buf);
      bool ok = wait_phase(bars + 8 * (C::B_S_FULL + buf), s_par[buf], abort_flag, lim,
                           (kRoleSoftmax << 8) | kSiteSFull);
      s_par[buf] ^= 1u;
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after_sync();

      uint32_t sr[128];
      tmem_ld128_sync(lane_base + s_col, sr);
      float sv[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(sr[c]);

      const bool need_mask = (p.causal && j >= ti.diag0 + s) || ((j + 1) * BN > p.N);
      if (need_mask) {
        const int lim_local = limit - j * BN;
#pragma unroll
        for (int c = 0; c < 128; ++c) sv[c] = (c < lim_local) ? sv[c] : -INFINITY;
      }
      float mx[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
      for (int c = 4; c < 124; c += 8) {
        mx[0] = max3(mx[0], sv[c], sv[c + 4]);
        mx[1] = max3(mx[1], sv[c + 1], sv[c + 5]);
        mx[2] = max3(mx[2], sv[c + 2], sv[c + 6]);
        mx[3] = max3(mx[3], sv[c + 3], sv[c + 7]);
      }
      const float m_blk =
          max3(max3(mx[0], mx[1], sv[124]), max3(mx[2], mx[3], sv[125]), fmaxf(sv[126], sv[127])) *
          sl2;

      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_ref = m_blk;
      } else if (m_blk > m_ref + kLazyRescaleLog2) {
        alpha = ex2(m_ref - m_blk);
        m_ref = m_blk;
        rescale = true;
      }
      const float neg_ref = (m_ref == -INFINITY) ? 0.f : -m_ref;

      if (j > 0) {
        // O must hold every earlier P V product before it is rescaled.
        ok = wait_phase(bars + 8 * (C::B_O_DONE + bar_idx), o_par, abort_flag, lim,
                        (kRoleSoftmax << 8) | kSiteODone);
        o_par ^= 1u;
        if (!__all_sync(0xffffffffu, ok)) return;
        tc_fence_after_sync();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int c = 0; c < HD; c += 16) {
            uint32_t ov[16];
            tmem_ld16_sync(lane_base + o_col + c, ov);
#pragma unroll
            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st16(lane_base + o_col + c, ov);
          }
        }
      }

      // P (128 x 16-bit per row = 64 columns) goes over the start of the S
      // buffer, handed to the MMA warp in two halves of 64 keys.
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = half * 64 + c * 32;
          uint32_t pk[16];
          if (need_mask)
            softmax_chunk<BF16, 0>(sv + col, sl2, neg_ref, pk, acc);
          else
            softmax_chunk<BF16, kPolyPairsPer8>(sv + col, sl2, neg_ref, pk, acc);
          tmem_st16(lane_base + s_col + col / 2, pk);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * (C::B_P_FULL + 2 * bar_idx + half));
      }
      l = l * alpha + (acc.x + acc.y);
      ++s_iter;
    }

    // Epilogue: wait for the last P V product, then O / l and the logsumexp.
    bool ok = wait_phase(bars + 8 * (C::B_O_DONE + bar_idx), o_par, abort_flag, lim,
                         (kRoleSoftmax << 8) | kSiteODone);
    o_par ^= 1u;
    if (!__all_sync(0xffffffffu, ok)) return;
    tc_fence_after_sync();
    const float inv_l = 1.f / l;
    T* orow = reinterpret_cast<T*>(p.o) + ti.b * p.o_stride_b + ti.h * p.o_stride_h +
              static_cast<long long>(row) * p.o_stride_n;
#pragma unroll 1
    for (int c = 0; c < HD; c += 32) {
      uint32_t ov[32];
      tmem_ld32_sync(lane_base + o_col + c, ov);
      uint4 w[4];
      uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        wp[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
      if (row < p.N) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = w[i];
      }
    }
    if (p.lse != nullptr && row < p.N)
      p.lse[(static_cast<long long>(ti.b) * p.H + ti.h) * p.N + row] =
          (m_ref + log2f(l)) * 0.69314718055994530942f;
    // The next tile's first P V overwrites O only after this group's next
    // p_full arrival, which comes after these loads completed.
    tc_fence_before_sync();
  }
}

template <int HD, int QS, int KVS, bool BF16>
__global__ void __launch_bounds__(FwdCfg<HD, QS, KVS, BF16>::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<HD, QS, KVS, BF16>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  const uint32_t bars = base + C::BAR_OFF;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * C::B_Q_FULL, 1);
    mbar_init(bars + 8 * C::B_Q_EMPTY, 1);
    for (int i = 0; i < KVS; ++i) {
      mbar_init(bars + 8 * (C::B_KV_FULL + i), 1);
      mbar_init(bars + 8 * (C::B_KV_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars + 8 * (C::B_S_FULL + i), 1);
      mbar_init(bars + 8 * (C::B_O_DONE + i), 1);
    }
    for (int i = 0; i < 4; ++i)  // [Q tile][half of P]: one arrival per softmax warp
      mbar_init(bars + 8 * (C::B_P_FULL + i), 4);
    mbar_init(bars + 8 * C::B_DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&p.tmap_q);
    tma_prefetch_desc(&p.tmap_k);
    tma_prefetch_desc(&p.tmap_v);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp < C::SOFTMAX_WARPS) {
    softmax_role<HD, QS, KVS, BF16>(p, base, tmem, abort_flag);
  } else if (warp == C::PRODUCER_WARP) {
    if (lane == 0) producer_role<HD, QS, KVS, BF16>(p, base, abort_flag);
  } else if (warp == C::MMA_WARP) {
    if (lane == 0) mma_role<HD, QS, KVS, BF16>(p, base, tmem, abort_flag);
  }  // the remaining warps of the last warpgroup have no role

  tc_fence_before_sync();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// One warp waits on an mbarrier nobody arrives at; the bounded wait must give
// up after `limit_ns`, record its code and return.  Exercises the watchdog
// path without any real hang.
__global__ void watchdog_selftest_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_word = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    wait_phase(smem_u32(&bar), 0, &abort_word, limit_ns, (kRoleTest << 8) | kSiteSelfTest);
  __syncthreads();
}

// Evaluates exp2_poly2 on n arguments (test hook for the software exp2).
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

}  // namespace fa_sm100
