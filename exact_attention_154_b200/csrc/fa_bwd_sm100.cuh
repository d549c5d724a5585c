// fa_bwd_sm100.cuh -- attention backward (dQ, dK, dV) for sm_100a.
//
// Gradient of the forward in fa_fwd_sm100.cuh for an upstream gradient dO.
// The score tile is recomputed from Q, K and the forward's per-row logsumexp
// (the recomputation the pages describe for the backward pass of the
// "Windows下RTX 3090编译Flash Attention 2.8.3全指南" page, sections 1 and 7);
// everything else follows from the chain rule through the forward:
//
//   D_i     = sum_c dO[i,c] * O[i,c]                     (bwd_dsum_kernel)
//   P[i,j]  = exp2(s_ij * scale * log2 e - LSE_i * log2 e)   visible keys
//   dV[j]   = sum_i P[i,j] dO[i]
//   dP[i,j] = dO[i] . V[j]
//   dS[i,j] = P[i,j] (dP[i,j] - D_i)
//   dK[j]   = scale * sum_i dS[i,j] Q[i]                 (bwd_dkdv_kernel)
//   dQ[i]   = scale * sum_j dS[i,j] K[j]                 (bwd_dq_kernel)
//
// Both kernels run on a persistent grid (min(units, SMs) CTAs taking units in
// turn); a unit is one resident 128-row block of one (b, h).
//
// bwd_dkdv_kernel: a unit per 128-key block j.  For every query block i it
// computes S^T = K_j Q_i^T and dP^T = V_j dO_i^T into TMEM (tcgen05, SS),
// forms P^T and dS^T in 16 bits (one thread per key row) and writes them back
// into TMEM over the dP^T columns it has read, and accumulates
// dV_j += P^T dO_i and dK_j += dS^T Q_i in TMEM with P^T and dS^T as TMEM
// operands (tcgen05.mma with A in tensor memory).  The S^T columns are free
// once read, so S^T for query block i+1 runs during block i's element work.
// bwd_dq_kernel: a unit per 128-query block i; recomputes S and dP the same
// way for every key block j and accumulates dQ_i += dS K_j in TMEM.
// Keeping the 16-bit tiles in TMEM leaves shared memory for five streamed
// tiles (three of Q / K, two of dO / V), so the blocks after this one load
// while it is computed.
//
// Roles per CTA (576 threads): warps 0-15 compute P and dS (thread = TMEM
// lane = tile row; warpgroup g takes columns 32 g .. 32 g + 31 of each
// block), warp 16 streams tiles with TMA, warp 17 owns TMEM and one of its
// threads issues every tcgen05.mma.  All mbarrier waits are bounded
// (wait_phase).
#pragma once

#include "fa_fwd_sm100.cuh"

namespace fa_sm100 {

struct BwdParams {
  CUtensorMap tmap_q;   // 4-D (d, N, H, B) views, box 64 elements x 128 rows
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  CUtensorMap tmap_do;
  const void* o;        // forward output [B, H, N, d]
  const void* dout;     // upstream gradient [B, H, N, d]
  const float* lse;     // forward logsumexp [B, H, N] (natural log)
  float* dsum;          // workspace [B, H, N]: D_i
  void* dq;             // outputs [B, H, N, d]
  void* dk;
  void* dv;
  int B, H, N, causal;
  float scale;
  float scale_log2;     // scale * log2(e)
  int nblk;             // 128-row blocks per (b, h)
  int units;            // B * H * nblk: one unit = one resident key (dK/dV) or query (dQ) block
  int out_vec32;        // dq, dk, dv 32-byte aligned: the epilogue writes whole 32-byte sectors
  unsigned long long wait_limit_ns;
};

template <int HD, bool KV>
struct BwdCfg {
  static_assert(HD == 64 || HD == 128, "backward head dim");
  static constexpr int CHUNKS = HD / 64;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;   // one [128 x HD] 16-bit tile
  // four compute warpgroups (key/query rows x 32 of the 128 columns each),
  // then the producer warp and the MMA warp.  The element work of a block
  // sits between its S / dP products and its accumulating products, so the
  // more warps share it the shorter that gap.
  static constexpr int COMPUTE_WARPS = 16;
  static constexpr int GROUP_COLS = 128 / (COMPUTE_WARPS / 4);
  static_assert(GROUP_COLS == 32, "a warp's columns: one per lane");
  static constexpr int THREADS = 32 * (COMPUTE_WARPS + 2);
  static constexpr int PRODUCER_WARP = COMPUTE_WARPS, MMA_WARP = COMPUTE_WARPS + 1;
  // Shared memory: the resident pair (K, V for dK/dV; Q, dO for dQ), two
  // rings of streamed tiles, barriers.  The A stream (Q for dK/dV, K for dQ)
  // is the B operand of S and of the last accumulating product (dK / dQ), so
  // a slot is held to the end of its step: three slots.  The B stream (dO /
  // V) is the B operand of dP (and of dV), released earlier: two slots.  With
  // two streamed steps in flight the next step's S can be issued during this
  // step's element work without waiting for its load.
  static constexpr int A_SLOTS = 3, B_SLOTS = 2;
  static constexpr int B_RES_FULL = 0, B_A_FULL = 1 /* [A slot] */, B_A_EMPTY = 4,
                       B_B_FULL = 7 /* [B slot] */, B_B_EMPTY = 9, B_SD_FULL = 11,
                       // per block, one arrival per compute warp: S (S^T) and dP (dP^T)
                       // read out of TMEM; P^T written (dK/dV only); dS (dS^T) written.
                       // P_FULL and DS_FULL have one barrier per block parity: with two dP
                       // regions the next block's S and dP are in while this block's
                       // element work runs, so a warp can arrive for block it+1 before
                       // another has arrived for block it (never for it+2: that needs
                       // every warp to have read block it+1's S).
                       B_S_READ = 12, B_P_FULL = 13 /* [2] */, B_DS_FULL = 15 /* [2] */,
                       B_DONE = 17, B_DRAIN = 18,
                       // the resident pair's last readers (a unit's last S and dP) ended
                       B_RES_EMPTY = 19, NUM_BARS = 20;
  static constexpr int SA_OFF = 0;                            // K (dkdv) / Q (dq)
  static constexpr int SB_OFF = TILE_BYTES;                   // V (dkdv) / dO (dq)
  static constexpr int RA_OFF = 2 * TILE_BYTES;               // A ring: Q (dkdv) / K (dq)
  static constexpr int RB_OFF = RA_OFF + A_SLOTS * TILE_BYTES;  // B ring: dO (dkdv) / V (dq)
  static constexpr int BAR_OFF = RB_OFF + B_SLOTS * TILE_BYTES;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int END_OFF = MISC_OFF + 16;
  // slack to align the base to 1024: the dynamic shared memory base is 16-byte
  // aligned, so at most 1008 bytes are skipped
  static constexpr int SMEM_BYTES = END_OFF + 1008;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // TMEM columns: S (or S^T), dP (or dP^T), then the accumulators.  The
  // 16-bit tiles go into the dP (dP^T) columns only, each compute group over
  // the 32 columns it has read itself: columns [32 g, 32 g + 16) of the dP
  // region hold P^T (dK/dV kernel), columns [32 g + 16, 32 g + 32) dS (dS^T),
  // packed two per column, for tile columns [32 g, 32 g + 32).  The S region
  // is free as soon as it has been read, so the next block's S product runs
  // while this block's element work does.
  // Where the accumulators leave 128 columns (the dQ kernel; the dK/dV kernel
  // at d = 64) there are two dP regions, used by alternate blocks: the next
  // block's dP is then issued with its S, before this block's accumulating
  // products have read this block's packed tiles.
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0, DP_COL = 128, ACC0_COL = 256, ACC1_COL = 256 + HD;
  static constexpr int DP_BUFS = (KV ? 256 + 2 * HD : 256 + HD) + 128 <= 512 ? 2 : 1;
  static constexpr uint32_t DP2_COL = KV ? 256 + 2 * HD : 256 + HD;
  __host__ __device__ static constexpr uint32_t dp_col(int it) {
    return (DP_BUFS == 2 && (it & 1)) ? DP2_COL : DP_COL;
  }
  // TMEM column of the packed 16-bit P^T / dS operand for MMA K-step kk (16
  // columns of the tile, 8 packed TMEM columns) of step it
  __host__ __device__ static constexpr uint32_t p_col(int it, int kk) {
    return dp_col(it) + 32u * static_cast<uint32_t>(kk / 2) + 8u * static_cast<uint32_t>(kk % 2);
  }
  __host__ __device__ static constexpr uint32_t ds_col(int it, int kk) { return p_col(it, kk) + 16u; }
};

// D_i = dO_i . O_i in fp32: HD / 8 threads per row, each one 16-byte load of
// O and of dO (8 values), summed across the row's threads by shuffles.
template <int HD, bool BF16>
__global__ void __launch_bounds__(256) bwd_dsum_kernel(const void* __restrict__ o,
                                                       const void* __restrict__ dout,
                                                       float* __restrict__ dsum, long long rows) {
  using T2 = typename std::conditional<BF16, __nv_bfloat162, __half2>::type;
  constexpr int TPR = HD / 8;     // threads per row
  constexpr int RPB = 256 / TPR;  // rows per block
  const long long row = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *(reinterpret_cast<const uint4*>(o) + row * TPR + part);
    const uint4 d = *(reinterpret_cast<const uint4*>(dout) + row * TPR + part);
    const T2* a2 = reinterpret_cast<const T2*>(&a);
    const T2* d2 = reinterpret_cast<const T2*>(&d);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 x, y;
      if constexpr (BF16) {
        x = __bfloat1622float2(a2[i]);
        y = __bfloat1622float2(d2[i]);
      } else {
        x = __half22float2(a2[i]);
        y = __half22float2(d2[i]);
      }
      acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
    }
  }
  // every lane takes part in the shuffles; a row's threads are TPR adjacent lanes
#pragma unroll
  for (int sh = TPR / 2; sh > 0; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
  if (row < rows && part == 0) dsum[row] = acc;
}

// Of every 8 argument pairs of P, how many take the FMA-pipe exp2 (exp2_poly2)
// instead of ex2.  Measured on B200 at d = 128 and 64: 1 of 8 no change, 2 and
// 3 of 8 slower (the exponential unit does not bound these kernels), so none.
#ifdef FA_BWD_POLY8
constexpr int BWD_POLY8 = FA_BWD_POLY8;
#else
constexpr int BWD_POLY8 = 0;
#endif

// Loads one [128 x HD] tile of a 4-D tensor map into shared memory.
template <int HD>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                          int row0, int h, int b) {
#pragma unroll
  for (int c = 0; c < HD / 64; ++c)
    tma_load_4d(dst + c * (128 * 128), map, bar, c * 64, row0, h, b);
}

// Writes NC (16 or 32) fp32 accumulator columns of one row (times `mul`) as
// 16-bit values: 32-byte stores when the row is 32-byte aligned (each fills
// whole L2 sectors: a 16-byte store from every lane of a warp touches 32 rows
// with half-sector writes, twice the transactions and a read-modify-write of
// each sector), else 16-byte stores.
template <bool BF16, int NC>
__device__ __forceinline__ void store_acc(void* dst_row, const uint32_t* acc, float mul, bool vec32) {
  uint4 w[NC / 8];
  uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
  for (int i = 0; i < NC / 2; ++i)
    wp[i] = pack2<BF16>(__uint_as_float(acc[2 * i]) * mul, __uint_as_float(acc[2 * i + 1]) * mul);
  if (vec32) {
#pragma unroll
    for (int i = 0; i < NC / 16; ++i) st_global_v8(static_cast<uint4*>(dst_row) + 2 * i, wp + 8 * i);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(dst_row);
#pragma unroll
    for (int i = 0; i < NC / 8; ++i) dst[i] = w[i];
  }
}

// One unit of work: a resident key block (dK/dV) or query block (dQ) of one
// (b, h), and the streamed blocks it meets.
struct BwdUnit {
  int bh, blk, b, h;
  int first, count;  // streamed blocks first .. first + count - 1
};

// Units in the order they are handed out.  Non-causal: (b, h)-major, so the
// units running at once share a head's streamed tiles in L2.  Causal: the
// units with the most blocks first (key block 0 of every head for dK/dV, the
// last query block for dQ), so that with the snake hand-out below the
// persistent CTAs get equal work.
__device__ __forceinline__ BwdUnit bwd_unit(const BwdParams& p, int u, bool kv) {
  BwdUnit w;
  if (p.causal) {
    const int nbh = p.B * p.H;
    const int rank = u / nbh;
    w.bh = u - rank * nbh;
    w.blk = kv ? rank : p.nblk - 1 - rank;
  } else {
    w.bh = u / p.nblk;
    w.blk = u - w.bh * p.nblk;
  }
  w.b = w.bh / p.H;
  w.h = w.bh - w.b * p.H;
  // causal: key block j meets query blocks j .. nblk-1, query block i meets
  // key blocks 0 .. i
  w.first = (kv && p.causal) ? w.blk : 0;
  const int last = (!kv && p.causal) ? w.blk : p.nblk - 1;
  w.count = last - w.first + 1;
  return w;
}

// Persistent hand-out: round r gives CTA c unit r * G + c, in reverse CTA
// order on odd rounds.
__device__ __forceinline__ int bwd_unit_of(int round, int cta, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

// KV = true: the dK/dV kernel (units: key blocks, streams Q and dO).
// KV = false: the dQ kernel (units: query blocks, streams K and V).
// Persistent: min(units, SMs) CTAs, each taking units in turn; every role
// counts the streamed steps over all its units, so ring slots and per-step
// barrier phases run on across units.
template <int HD, bool BF16, bool KV>
__global__ void __launch_bounds__(BwdCfg<HD, KV>::THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<HD, KV>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  const uint32_t bars = base + C::BAR_OFF;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const unsigned long long lim = p.wait_limit_ns;

  const int G = gridDim.x, cta = blockIdx.x;

  if (threadIdx.x == 0) {
    // S read, P written, dS written: one arrival per compute warp; the rest
    // are single
    for (int i = 0; i < C::NUM_BARS; ++i)
      mbar_init(bars + 8 * i, (i >= C::B_S_READ && i < C::B_DONE) ? C::COMPUTE_WARPS : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&p.tmap_q);
    tma_prefetch_desc(&p.tmap_k);
    tma_prefetch_desc(&p.tmap_v);
    tma_prefetch_desc(&p.tmap_do);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp == C::PRODUCER_WARP) {
    if (lane == 0) {
      bool ok = true;
      int g = 0, k = 0;                // streamed steps and units so far
      int issued_a = 0, issued_b = 0;  // ring loads issued (= g after each unit)
      for (int round = 0; ok && round * G < p.units; ++round) {
        const int u = bwd_unit_of(round, cta, G);
        if (u >= p.units) continue;
        const BwdUnit w = bwd_unit(p, u, KV);
        // resident pair: K_j, V_j (dkdv) or Q_i, dO_i (dq), once the previous
        // unit's S and dP products have ended
        if (k > 0 && !(ok = wait_phase(bars + 8 * C::B_RES_EMPTY, (k - 1) & 1, abort_flag, lim,
                                       (kRoleProducer << 8) | kSiteQEmpty)))
          break;
        mbar_arrive_expect_tx(bars + 8 * C::B_RES_FULL, 2 * C::TILE_BYTES);
        load_tile<HD>(base + C::SA_OFF, KV ? &p.tmap_k : &p.tmap_q, bars + 8 * C::B_RES_FULL,
                      w.blk * 128, w.h, w.b);
        load_tile<HD>(base + C::SB_OFF, KV ? &p.tmap_v : &p.tmap_do, bars + 8 * C::B_RES_FULL,
                      w.blk * 128, w.h, w.b);
        ++k;
        // A_it then B_it, each into its ring once the slot's previous tile is
        // released
        for (int it = 0; ok && it < w.count; ++it) {
          const int gs = g + it, row0 = (w.first + it) * 128;
#pragma unroll 1
          for (int ring = 0; ring < 2; ++ring) {
            const int slots = ring ? C::B_SLOTS : C::A_SLOTS;
            const int slot = gs % slots, use = gs / slots;
            const int b_empty = ring ? C::B_B_EMPTY : C::B_A_EMPTY;
            if (use > 0 && !(ok = wait_phase(bars + 8 * (b_empty + slot), (use - 1) & 1, abort_flag,
                                             lim, (kRoleProducer << 8) | kSiteKvEmpty)))
              break;
            const uint32_t full = bars + 8 * ((ring ? C::B_B_FULL : C::B_A_FULL) + slot);
            mbar_arrive_expect_tx(full, C::TILE_BYTES);
            load_tile<HD>(base + (ring ? C::RB_OFF : C::RA_OFF) + slot * C::TILE_BYTES,
                          ring ? (KV ? &p.tmap_do : &p.tmap_v) : (KV ? &p.tmap_q : &p.tmap_k),
                          full, row0, w.h, w.b);
            ++(ring ? issued_b : issued_a);
          }
        }
        g += w.count;
      }
      if (!ok) {
        // let the loads in flight land before the shared memory goes away
        volatile int no_abort = 0;
        if (k > 0)
          wait_phase(bars + 8 * C::B_RES_FULL, (k - 1) & 1, &no_abort, 10000000ull,
                     (kRoleProducer << 8) | kSiteDrain);
        for (int i = issued_a > C::A_SLOTS ? issued_a - C::A_SLOTS : 0; i < issued_a; ++i)
          wait_phase(bars + 8 * (C::B_A_FULL + i % C::A_SLOTS), (i / C::A_SLOTS) & 1, &no_abort,
                     10000000ull, (kRoleProducer << 8) | kSiteDrain);
        for (int i = issued_b > C::B_SLOTS ? issued_b - C::B_SLOTS : 0; i < issued_b; ++i)
          wait_phase(bars + 8 * (C::B_B_FULL + i % C::B_SLOTS), (i / C::B_SLOTS) & 1, &no_abort,
                     10000000ull, (kRoleProducer << 8) | kSiteDrain);
      }
    }
  } else if (warp == C::MMA_WARP) {
    if (lane == 0) {
      const uint32_t idesc_sq = f16_idesc(BF16, 128, 128, false);  // S-shaped: N = 128 rows
      const uint32_t idesc_acc = f16_idesc(BF16, 128, HD, true);   // accumulators: N = HD
      bool ok = true;
      // K-major [128 x HD] operands: resident A-side tiles ...
      const uint32_t a0 = sw128_desc_lo(base + C::SA_OFF, 16), a1 = sw128_desc_lo(base + C::SB_OFF, 16);
      // the streamed tiles of global step gs: K-major B of S (A ring) / dP (B
      // ring), MN-major B [K = 128 rows x N = HD] of the accumulating products
      // (Q for dK, K for dQ from the A ring; dO for dV from the B ring)
      auto ra = [&](int gs) { return base + C::RA_OFF + (gs % C::A_SLOTS) * C::TILE_BYTES; };
      auto rb = [&](int gs) { return base + C::RB_OFF + (gs % C::B_SLOTS) * C::TILE_BYTES; };
      auto wait_ring = [&](int gs, int ring) -> bool {
        const int slots = ring ? C::B_SLOTS : C::A_SLOTS;
        const bool r = wait_phase(bars + 8 * ((ring ? C::B_B_FULL : C::B_A_FULL) + gs % slots),
                                  (gs / slots) & 1, abort_flag, lim, (kRoleMma << 8) | kSiteKvFull);
        tc_fence_after_sync();
        return r;
      };
      // dkdv: S^T = K Q^T (a0, A ring), dP^T = V dO^T (a1, B ring);
      // dq: S = Q K^T, dP = dO V^T
      auto issue_sq = [&](uint32_t d_col, uint32_t a, uint32_t bt) {
        const uint32_t bd = sw128_desc_lo(bt, 16);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = ((kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32) >> 4;
          mma_ss(tmem + d_col, desc_from_lo(a + off), desc_from_lo(bd + off), idesc_sq,
                 kk > 0 ? 1u : 0u);
        }
      };
      // dP of step gs; in the dQ kernel the B-ring tile (V) has no other use
      auto issue_dp = [&](int gs) {
        issue_sq(C::dp_col(gs), a1, rb(gs));
        tc_commit(bars + 8 * C::B_SD_FULL);
        if (!KV) tc_commit(bars + 8 * (C::B_B_EMPTY + gs % C::B_SLOTS));
      };
      int g = 0, k = 0;  // streamed steps and units so far
      for (int round = 0; ok && round * G < p.units; ++round) {
        const int u = bwd_unit_of(round, cta, G);
        if (u >= p.units) continue;
        const int count = bwd_unit(p, u, KV).count;
        // The unit's resident pair.  (The previous unit's last S was read out
        // before its last dK / dQ, which waited for every warp's dS of that
        // step; its accumulators are read out by each warp's epilogue before
        // that warp's P / dS of this unit's first step, which this unit's
        // first accumulating products wait for.)
        if (!(ok = wait_phase(bars + 8 * C::B_RES_FULL, k & 1, abort_flag, lim,
                              (kRoleMma << 8) | kSiteQFull)))
          break;
        tc_fence_after_sync();
        ++k;
        if (!(ok = wait_ring(g, 0))) break;
        issue_sq(C::S_COL, a0, ra(g));
        if (!(ok = wait_ring(g, 1))) break;
        issue_dp(g);
        // the resident pair is free once the unit's last S and dP have ended
        if (count == 1) tc_commit(bars + 8 * C::B_RES_EMPTY);
        // Per step: the next S once this step's S has been read out (and with
        // two dP regions the next dP with it: its region's last packed tiles
        // were read by products issued before); the accumulating products once
        // their 16-bit operand is written; with one dP region the next dP after
        // them (its columns hold that operand until they have read it:
        // tcgen05.mma operations from one thread run in issue order).
        for (int it = 0; ok && it < count; ++it) {
          const int gs = g + it;
          const uint32_t mq = sw128_desc_lo(ra(gs), C::CHUNK_BYTES);
          const uint32_t md = sw128_desc_lo(rb(gs), C::CHUNK_BYTES);
          const bool more = it + 1 < count;
          if (more) {
            if (!(ok = wait_ring(gs + 1, 0))) break;
            if (!(ok = wait_phase(bars + 8 * C::B_S_READ, gs & 1, abort_flag, lim,
                                  (kRoleMma << 8) | kSiteSFree)))
              break;
            tc_fence_after_sync();
            issue_sq(C::S_COL, a0, ra(gs + 1));
            if (C::DP_BUFS == 2) {
              if (!(ok = wait_ring(gs + 1, 1))) break;
              issue_dp(gs + 1);
              if (it + 2 == count) tc_commit(bars + 8 * C::B_RES_EMPTY);
            }
          }
          if (KV) {
            // dV += P^T dO; then dO's slot is free
            if (!(ok = wait_phase(bars + 8 * (C::B_P_FULL + (gs & 1)), (gs >> 1) & 1, abort_flag,
                                  lim, (kRoleMma << 8) | kSitePFull)))
              break;
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + C::ACC0_COL, tmem + C::p_col(gs, kk),
                     desc_from_lo(md + ((kk * 16 * 128) >> 4)), idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
            tc_commit(bars + 8 * (C::B_B_EMPTY + gs % C::B_SLOTS));
          }
          // dK += dS^T Q (dkdv) or dQ += dS K (dq); then the A slot is free
          if (!(ok = wait_phase(bars + 8 * (C::B_DS_FULL + (gs & 1)), (gs >> 1) & 1, abort_flag, lim,
                                (kRoleMma << 8) | kSitePFull)))
            break;
          tc_fence_after_sync();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + (KV ? C::ACC1_COL : C::ACC0_COL), tmem + C::ds_col(gs, kk),
                   desc_from_lo(mq + ((kk * 16 * 128) >> 4)), idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bars + 8 * (C::B_A_EMPTY + gs % C::A_SLOTS));
          if (more && C::DP_BUFS == 1) {
            if (!(ok = wait_ring(gs + 1, 1))) break;
            issue_dp(gs + 1);
            if (it + 2 == count) tc_commit(bars + 8 * C::B_RES_EMPTY);
          }
        }
        if (!ok) break;
        // the unit's accumulators are complete once these products end
        tc_commit(bars + 8 * C::B_DONE);
        g += count;
      }
      if (!ok) {
        // wait for every MMA this thread issued before TMEM is released
        volatile int no_abort = 0;
        tc_commit(bars + 8 * C::B_DRAIN);
        wait_phase(bars + 8 * C::B_DRAIN, 0, &no_abort, 10000000ull, (kRoleMma << 8) | kSiteDrain);
      }
    }
  } else {
    // compute warps: thread = tile row = TMEM lane; this warpgroup's columns
    constexpr int GC = C::GROUP_COLS;
    static_assert(GC == 32, "one 32-column pass per block");
    const int quad = warp % 4, grp = warp / 4, cb = GC * grp;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = tmem + ((static_cast<uint32_t>(quad) * 32u) << 16);
    const float sl2 = p.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    bool ok = true;
    int g = 0, k = 0;  // streamed steps and units so far
    for (int round = 0; ok && round * G < p.units; ++round) {
      const int u = bwd_unit_of(round, cta, G);
      if (u >= p.units) continue;
      const BwdUnit w = bwd_unit(p, u, KV);
      const long long vec0 = static_cast<long long>(w.bh) * p.N;
      const int my_row = w.blk * 128 + r;  // key row (dkdv) or query row (dq)
      float my_lse2 = INFINITY, my_dsum = 0.f;
      if (!KV && my_row < p.N) {
        my_lse2 = p.lse[vec0 + my_row] * kLog2e;
        my_dsum = p.dsum[vec0 + my_row];
      }
      for (int it = 0; it < w.count; ++it) {
        const int gs = g + it;
        const int other0 = (w.first + it) * 128;  // first streamed row of this step
        // dkdv: the statistics of the streamed query block's columns, lane l
        // holding column cb + l (+inf lse masks query rows past N); read by
        // shuffles below
        float col_lse2 = INFINITY, col_dsum = 0.f;
        if (KV) {
          const int qi = other0 + cb + lane;
          if (qi < p.N) {
            col_lse2 = p.lse[vec0 + qi] * kLog2e;
            col_dsum = p.dsum[vec0 + qi];
          }
        }
        ok = wait_phase(bars + 8 * C::B_SD_FULL, gs & 1, abort_flag, lim,
                        (kRoleSoftmax << 8) | kSiteSFull);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after_sync();
        // (the 16-bit tiles last written to this step's dP columns were read by
        // products that the MMA thread issued before this step's dP)
        // S and dP of this thread's row over the group's 32 columns, one wait
        uint32_t sd[64];
        const uint32_t dpc = C::dp_col(gs);
        tmem_ld32x2_nowait(lane_base + C::S_COL + cb, lane_base + dpc + cb, sd);
        tmem_ld64_wait(sd);
        // both are in registers: the next S may overwrite the S columns
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * C::B_S_READ);
        // P (kept in fp32 over the S registers for dS); BWD_POLY8 of every 8
        // argument pairs take the FMA-pipe exp2, the rest ex2
        uint32_t pk[16];
  #pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float2 nl = KV ? make_float2(-__shfl_sync(0xffffffffu, col_lse2, 2 * q),
                                             -__shfl_sync(0xffffffffu, col_lse2, 2 * q + 1))
                               : make_float2(-my_lse2, -my_lse2);
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sd[2 * q]), __uint_as_float(sd[2 * q + 1])),
                                      make_float2(sl2, sl2), nl);
          float2 ev;
          if ((q % 8) >= 8 - BWD_POLY8) {
            ev = exp2_poly2(x);
          } else {
            ev.x = ex2(x.x);
            ev.y = ex2(x.y);
          }
          float pp[2] = {ev.x, ev.y};
  #pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = cb + 2 * q + e;
            // dkdv: row = key my_row, column = query other0 + c (columns past N
            // carry lse = +inf); dq: row = query my_row, column = key other0 + c
            const bool vis = KV ? (!p.causal || other0 + c >= my_row)
                                : (other0 + c < p.N && (!p.causal || other0 + c <= my_row));
            pp[e] = vis ? pp[e] : 0.f;
            sd[2 * q + e] = __float_as_uint(pp[e]);
          }
          pk[q] = pack2<BF16>(pp[0], pp[1]);
        }
        if (KV) {
          // P^T over the first 16 of the group's dP^T columns (read above)
          tmem_st16(lane_base + dpc + cb, pk);
          tmem_st_wait();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(bars + 8 * (C::B_P_FULL + (gs & 1)));
        }
        // dS = P (dP - D)
        uint32_t dk[16];
  #pragma unroll
        for (int q = 0; q < 16; ++q) {
          float ds[2];
  #pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = cb + 2 * q + e;
            const float pv = __uint_as_float(sd[2 * q + e]);
            const float dpv = __uint_as_float(sd[32 + 2 * q + e]);
            ds[e] = pv * (dpv - (KV ? __shfl_sync(0xffffffffu, col_dsum, c - cb) : my_dsum));
          }
          dk[q] = pack2<BF16>(ds[0], ds[1]);
        }
        // over the last 16 of the group's dP columns
        tmem_st16(lane_base + dpc + cb + 16, dk);
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * (C::B_DS_FULL + (gs & 1)));
      }
      if (ok) {
        ok = wait_phase(bars + 8 * C::B_DONE, k & 1, abort_flag, lim, (kRoleSoftmax << 8) | kSiteODone);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after_sync();
          using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
          const long long row_off = (vec0 + my_row) * HD;
          // this group's quarter of the accumulator columns
          constexpr int EC = HD / (C::COMPUTE_WARPS / 4);
          const bool vec32 = p.out_vec32 != 0;
          const int c = grp * EC;
          if constexpr (EC == 32) {
            uint32_t a0[32], a1[32];
            tmem_ld32_sync(lane_base + C::ACC0_COL + c, a0);
            if (KV) tmem_ld32_sync(lane_base + C::ACC1_COL + c, a1);
            if (my_row < p.N) {
              if (KV) {
                store_acc<BF16, 32>(static_cast<T*>(p.dv) + row_off + c, a0, 1.f, vec32);
                store_acc<BF16, 32>(static_cast<T*>(p.dk) + row_off + c, a1, p.scale, vec32);
              } else {
                store_acc<BF16, 32>(static_cast<T*>(p.dq) + row_off + c, a0, p.scale, vec32);
              }
            }
          } else {
            static_assert(EC == 16, "accumulator quarter");
            uint32_t a0[16], a1[16];
            tmem_ld16_sync(lane_base + C::ACC0_COL + c, a0);
            if (KV) tmem_ld16_sync(lane_base + C::ACC1_COL + c, a1);
            if (my_row < p.N) {
              if (KV) {
                store_acc<BF16, 16>(static_cast<T*>(p.dv) + row_off + c, a0, 1.f, vec32);
                store_acc<BF16, 16>(static_cast<T*>(p.dk) + row_off + c, a1, p.scale, vec32);
              } else {
                store_acc<BF16, 16>(static_cast<T*>(p.dq) + row_off + c, a0, p.scale, vec32);
              }
            }
          }
        }
      }
      g += w.count;
      ++k;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa_sm100
