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
//     full / empty mbarriers (128-byte swizzle; every CTA loads its own
//     tiles), K one block ahead of V;
//   * two threads issue the tcgen05 MMAs, one per product, because a thread
//     that issues MMAs runs only about one instruction ahead of the tensor
//     pipe: one issues S = Q K^T into tensor memory (TMEM), the other
//     O += P V with P from shared memory, each committing its groups to
//     mbarriers;
//   * two softmax warpgroups own each Q tile, one per 64 key columns: thread t
//     of a group owns query row t (TMEM lane t), so the row max and row sum
//     need no shuffles, only one exchange per block between the two groups
//     through shared memory.  Each group reads its half of S from TMEM and,
//     once the row max is agreed, releases the S buffer so the tensor core can
//     already compute the next block's S; then it applies scale (in the log2
//     domain), the causal / ragged mask and the online update, rescales its
//     half of O in TMEM when the reference max moved, writes its half of P as
//     16-bit values into the one shared-memory P tile the Q tiles use in turn
//     (handed over by 64-key halves), and finally writes its half of O / l
//     and (one group) the logsumexp.
//
// Because S(j+1) is computed while the softmax of block j runs, the softmax
// groups work back to back; four of them share each SM sub-partition, which
// hides the latency of the TMEM loads, the exponential unit and the hand-off
// fences that two alone leave exposed.
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
// Argument pairs (of every 8) whose exp2 runs on the FMA pipe instead of
// MUFU.  With two Q tiles (d = 64, 128) the exponentials are cheaper on MUFU
// alone; with one (d = 256) a quarter on the FMA pipe helps (measured).  A
// build may fix the number for every head dim.
template <int HD>
__host__ __device__ constexpr int poly_pairs_per8() {
#ifdef FA_POLY_PAIRS_PER8
  return FA_POLY_PAIRS_PER8;
#else
  return HD == 256 ? 2 : 0;
#endif
}

// Operand element types of the forward: fp16 and bf16 (kind::f16 MMAs, P and
// O in the same type) and fp8 e4m3 (kind::f8f6f4 MMAs, P in e4m3, O in bf16).
enum Elt : int { kF16 = 0, kBF16 = 1, kE4M3 = 2 };
__host__ __device__ constexpr int elt_bytes(int elt) { return elt == kE4M3 ? 1 : 2; }

// Error word written by a kernel whose bounded wait ran out: 0 = none,
// otherwise (role << 8) | site, first writer wins.
__device__ unsigned int g_fa_watchdog = 0u;

enum WaitSite : unsigned {
  kSiteQEmpty = 1, kSiteKvEmpty = 2, kSiteQFull = 3, kSiteKvFull = 4, kSitePFull = 5,
  kSiteSFull = 6, kSiteODone = 7, kSiteSelfTest = 8, kSiteDrain = 9, kSiteSFree = 10,
  kSitePFree = 11, kSiteAlign = 12, kSiteXch = 13, kSiteSeqlens = 14, kSiteOSlot = 15,
  kSiteOStaged = 16
};
// kRoleArgs: not a wait but a device-side argument check (cu_seqlens out of
// range); the offending work tile is skipped.
enum Role : unsigned {
  kRoleProducer = 1, kRoleMma = 2, kRoleSoftmax = 3, kRoleTest = 4, kRoleArgs = 5,
  kRoleStore = 6
};

struct FwdParams {
  // 4-D (d, rows, H, batches) views of q, k, v; box 64 elements x 128 rows.
  // Fixed-length problems: rows = N, batches = B.  Variable-length problems
  // (cu_seqlens != nullptr): rows = the packed token count, one batch.
  CUtensorMap tmap_q;
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  CUtensorMap tmap_o;  // the same view of o (16-bit outputs), for the TMA stores
  void* o;
  float* lse;  // nullptr, or indexed [bc * lse_stride_b + h * lse_stride_h + token row]
  long long o_stride_b, o_stride_h, o_stride_n;  // in elements
  long long lse_stride_b, lse_stride_h;
  int B, H, N;       // N: the sequence length, or the longest one when variable
  int rows_total;    // rows of the tensor maps (N, or the packed token count)
  const int* cu_seqlens;  // [B + 1] token offsets of the sequences, or nullptr
  int causal;
  // Key j is visible from query i iff i - window_left <= j <= i + window_right
  // (and j < the sequence length); -1 leaves that side unbounded.  The causal
  // mask arrives here as window_right = 0.
  int window_left, window_right;
  const float* alibi_slopes;  // [H]: the scaled score gets -slope[h] * |i - j|; or nullptr
  float scale_log2;  // scale * log2(e) (e4m3: times the q and k descale factors)
  float o_scale;     // factor on O / l: 1, or the v descale factor (e4m3)
  int o_vec32;       // o and its strides are 32-byte aligned: 32-byte stores
  int num_qblocks;   // query blocks per (b, h) (of the longest sequence)
  int num_tiles;     // B * H * num_qblocks
  unsigned long long wait_limit_ns;
};

// Bounded wait on an mbarrier phase.  Gives up when the CTA-wide abort flag
// is raised or after `limit_ns`; the first to give up records `code`.  Past
// the first try (the fast path) the time and the flag are checked after every
// try, so the bound holds to within one hardware suspension of the thread.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned long long limit_ns, unsigned code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicCAS(&g_fa_watchdog, 0u, code);
      return false;
    }
  }
}

template <int HD, int QS, int KVS, int ELT>
struct FwdCfg {
  static_assert(HD == 64 || HD == 128 || HD == 256, "head dim");
  static_assert(QS == 1 || QS == 2, "Q tiles per work tile");
  static_assert(ELT != kE4M3 || HD >= 128, "fp8 rows must fill a 128-byte swizzle row");
  static constexpr int EB = elt_bytes(ELT);         // bytes per element
  static constexpr int BOX = 128 / EB;              // elements per 128-byte row chunk
  static constexpr int CHUNKS = HD * EB / 128;      // 128-byte column chunks per row
  static constexpr int CHUNK_BYTES = 128 * 128;     // one chunk of a 128-row tile
  static constexpr int TILE_BYTES = CHUNKS * CHUNK_BYTES;
  // Every MMA K-step takes 32 bytes of each operand row: 16 fp16 / bf16 or
  // 32 e4m3 elements.
  static constexpr int KSTEP = 32 / EB;
  static constexpr int S_KSTEPS = HD / KSTEP;       // S = Q K^T
  static constexpr int PV_KSTEPS = BN / KSTEP;      // O += P V, over the 128 keys
  // one 128 x 128 P tile (16-bit, or e4m3), used by the Q tiles in turn
  static constexpr int P_TILE_BYTES = (BN * EB / 128) * CHUNK_BYTES;
  // two softmax warpgroups per Q tile: key columns 0-63 and 64-127 of the
  // same 128 rows
  static constexpr int SOFTMAX_WGS = 2 * QS;
  static constexpr int SOFTMAX_WARPS = 4 * SOFTMAX_WGS;
  static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;
  static constexpr int MMA_S_WARP = SOFTMAX_WARPS + 1;   // issues S = Q K^T, owns TMEM
  static constexpr int MMA_PV_WARP = SOFTMAX_WARPS + 2;  // issues O += P V
  static constexpr int STORE_WARP = SOFTMAX_WARPS + 3;   // TMA stores of O (16-bit outputs)
  // 16-bit outputs leave the SM by TMA stores from a K/V ring slot; the e4m3
  // path writes bf16 O, twice its slot, with per-thread stores, and so does
  // head dim 256, whose two-slot ring cannot spare a slot at a work tile's
  // end (measured 1-2% slower with it)
  static constexpr bool O_TMA = ELT != kE4M3 && HD != 256;
  // whole warpgroups: the softmax groups, then one group holding the producer
  // warp, the two MMA warps and one warp without a role
  static constexpr int THREADS = 128 * (SOFTMAX_WGS + 1);
  // With 640 threads the launch budget is 96 registers a thread; setmaxnreg
  // moves registers from the last warpgroup to the softmax groups:
  // 4 * 128 * 104 + 128 * 64 = 61440 = 640 * 96 (the build checks the 96).
  static constexpr bool REG_SPLIT = THREADS == 640;
  static constexpr int SOFTMAX_REGS = 104, OTHER_REGS = 64;

  static constexpr int SQ_OFF = 0;
  static constexpr int SP_OFF = QS * TILE_BYTES;
  static constexpr int SKV_OFF = SP_OFF + P_TILE_BYTES;
  static constexpr int BAR_OFF = SKV_OFF + KVS * TILE_BYTES;
  // barrier indices ([Q tile] unless noted).  A ring slot holds K, V or O
  // tiles in turn; its "full" barrier is split by consumer -- K loads complete
  // on B_K_FULL (the S thread), V loads on B_V_FULL (the P V thread), O
  // reservations on B_O_READY (the softmax groups) -- so every barrier has
  // one consumer that waits each of its phases in order.  (A parity wait only
  // tells a phase from the one before it: a shared barrier could be two
  // phases away from a consumer that skips the others' uses.)
  static constexpr int B_Q_FULL = 0, B_Q_EMPTY = 1, B_K_FULL = 2, B_V_FULL = 2 + KVS,
                       B_O_READY = 2 + 2 * KVS, B_KV_EMPTY = 2 + 3 * KVS,
                       B_S_FULL = 2 + 4 * KVS, B_S_FREE = B_S_FULL + 2,
                       B_P_FULL = B_S_FREE + 2,  // [half of P] of the tile using the buffer
                       B_P_FREE = B_P_FULL + 2,  // [Q tile][half]: that half is this tile's turn
                       B_PV_DONE = B_P_FREE + 4,  // [Q tile]: a P V product of the tile finished
                       B_O_FINAL = B_PV_DONE + 2,
                       B_XCH = B_O_FINAL + 2,  // the two softmax groups of a tile met
                       B_DRAIN = B_XCH + 2,    // [MMA thread]
                       // [ring slot]: a tile's O written into that slot.  One per slot,
                       // so that a slot's next O use -- which needs this one's release
                       // by the store warp -- cannot run a phase ahead of its waiter.
                       B_O_STAGED = B_DRAIN + 2,
                       NUM_BARS = B_O_STAGED + KVS;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int XCH_OFF = MISC_OFF + 16;  // row max / row sum exchange [tile][half][row]
  static constexpr int END_OFF = XCH_OFF + 2 * 2 * 128 * 4;
  static_assert(END_OFF <= 232448, "shared memory budget");
  // whatever is left up to the 227 KB limit pads the start to 1024 bytes
  static constexpr int ALIGN_SLACK = (232448 - END_OFF) < 1008 ? (232448 - END_OFF) : 1008;
  static constexpr int SMEM_BYTES = END_OFF + ALIGN_SLACK;

  // TMEM columns (fp32 words): one S buffer per Q tile, then the O accumulators.
  static constexpr uint32_t TMEM_COLS = 512;
  __host__ __device__ static constexpr uint32_t s_col(int tile) { return tile ? 128u : 0u; }
  static constexpr uint32_t O_COL0 = 256u;
  static constexpr uint32_t O_COL1 = 256u + HD;
  static_assert(128 * QS <= 256 && 256 + QS * HD <= 512, "TMEM budget");
};

// One work tile: up to two 128-row Q tiles of one (sequence, head).  Q tile s
// needs the key blocks [lo[s], hi[s]) (empty: lo == hi == 0); the work tile
// streams their union [lo_u, lo_u + n_u), which is contiguous because the Q
// tiles are adjacent and every row sees its own key.
struct TileInfo {
  int b, h, q0;  // q0: first query row, relative to the sequence
  int len;       // the sequence's length (queries = keys)
  int row0;      // tensor-map row of the sequence's first token
  int bc;        // tensor-map batch coordinate
  int lo[2], hi[2];
  int lo_u, n_u;
};

__device__ __forceinline__ bool in_range(const TileInfo& ti, int s, int j) {
  return j >= ti.lo[s] && j < ti.hi[s];
}

// Key blocks [lo, hi) a 128-row Q tile starting at row r0 of a sequence of
// `len` tokens needs: those holding a key visible from one of its rows (up to
// and including the diagonal block with the causal mask, the blocks the window
// reaches with a local window).
__device__ __forceinline__ void key_range(const FwdParams& p, int len, int r0, int& lo, int& hi) {
  if (r0 >= len) {
    lo = hi = 0;
    return;
  }
  const int nkv = (len + BN - 1) / BN;
  const int last_row = min(r0 + BM - 1, len - 1);
  lo = p.window_left < 0 ? 0 : max(0, r0 - p.window_left) / BN;
  hi = p.window_right < 0 ? nkv : min(len - 1, last_row + p.window_right) / BN + 1;
}

template <int QS>
__device__ __forceinline__ TileInfo decode_tile(const FwdParams& p, int t) {
  TileInfo ti;
  int bh, qblock;
  if (p.causal) {
    // longest first over the whole grid: all heads' last query block, then
    // the one before, ...; with the snake hand-out below this balances the
    // triangular work to within a few percent
    const int nbh = p.B * p.H;
    const int qi = t / nbh;
    bh = t - qi * nbh;
    qblock = p.num_qblocks - 1 - qi;
  } else {
    // equal work per tile: keep a head's query blocks together for K/V reuse in L2
    bh = t / p.num_qblocks;
    qblock = t - bh * p.num_qblocks;
  }
  ti.b = bh / p.H;
  ti.h = bh - ti.b * p.H;
  ti.q0 = qblock * BM * QS;
  if (p.cu_seqlens != nullptr) {
    const int s0 = __ldg(p.cu_seqlens + ti.b), s1 = __ldg(p.cu_seqlens + ti.b + 1);
    ti.row0 = s0;
    ti.len = s1 - s0;
    ti.bc = 0;
    if (s0 < 0 || ti.len < 0 || ti.len > p.N || s1 > p.rows_total) {
      // offsets out of range: skip the tile and report it (only one role does)
      if (threadIdx.x == 0) atomicCAS(&g_fa_watchdog, 0u, (kRoleArgs << 8) | kSiteSeqlens);
      ti.len = 0;
    }
  } else {
    ti.row0 = 0;
    ti.len = p.N;
    ti.bc = ti.b;
  }
  key_range(p, ti.len, ti.q0, ti.lo[0], ti.hi[0]);
  if (QS == 2)
    key_range(p, ti.len, ti.q0 + BM, ti.lo[1], ti.hi[1]);
  else
    ti.lo[1] = ti.hi[1] = 0;
  ti.lo_u = ti.lo[0];
  ti.n_u = ti.hi[0] == 0 ? 0 : max(ti.hi[0], ti.hi[1]) - ti.lo[0];
  return ti;
}

// Ring positions (from the work tile's first) of K(j) and V(j) when a work
// tile streams K(0), then K(j+1), V(j) for j = 0 .. n-2, then V(n-1): each K
// tile is requested before the V tile of the block before it, so a K load
// never queues behind a V slot that the slower P V has yet to release.
__host__ __device__ __forceinline__ int ring_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__host__ __device__ __forceinline__ int ring_v(int j, int n) { return j < n - 1 ? 2 * j + 2 : 2 * n - 1; }

// Order in which the Q tiles of a work tile use the shared P buffer: block j
// of tile 0 (if in its range), then block j of tile 1 (likewise), then block
// j + 1, ...  Tile 0's range starts first, so it is every work tile's first
// user.  Returns the tile of the use after (s, j), or -1 if (s, j) is the
// work tile's last.
__device__ __forceinline__ int next_p_user(int s, int j, const TileInfo& ti) {
  if (s == 0 && in_range(ti, 1, j)) return 1;
  if (in_range(ti, 0, j + 1)) return 0;
  if (in_range(ti, 1, j + 1)) return 1;
  return -1;
}

// O of Q tile s leaves through a K/V ring slot (staged by the softmax groups,
// stored by TMA) when the output is 16-bit, the tile is not empty and -- for
// packed variable-length sequences, where a box past the sequence's end would
// write the next sequence's rows -- the whole 128-row box lies inside the
// sequence.  Such tiles take one ring position each after the work tile's
// last V: position 2 n_u for the first, 2 n_u + 1 for the second.
template <bool O_TMA>
__device__ __forceinline__ bool o_via_slot(const FwdParams& p, const TileInfo& ti, int s) {
  if (!O_TMA || ti.lo[s] == ti.hi[s]) return false;
  return p.cu_seqlens == nullptr || ti.q0 + (s + 1) * BM <= ti.len;
}
template <bool O_TMA>
__device__ __forceinline__ int o_slots(const FwdParams& p, const TileInfo& ti) {
  return (o_via_slot<O_TMA>(p, ti, 0) ? 1 : 0) + (o_via_slot<O_TMA>(p, ti, 1) ? 1 : 0);
}

// Static persistent schedule: round r hands tiles [r*G, (r+1)*G) to the G
// CTAs, reversing the order on odd rounds, so that with the longest-first
// causal order every CTA gets a long and a short tile in each pair of rounds.
__device__ __forceinline__ int tile_of(int round, int cta, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

// Two e4m3 codes (round to nearest, saturating) in 16 bits: lo in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
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
template <int HD, int QS, int KVS, int ELT>
__device__ void producer_role(const FwdParams& p, uint32_t base, volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, ELT>;
  const uint32_t bars = base + C::BAR_OFF;
  const int G = gridDim.x, cta = blockIdx.x;
  int kv_count = 0, q_count = 0;
  bool ok = true;
  // For the drain after an abort: the last load into each slot (its barrier
  // and the parity of the phase it completes).
  uint32_t k_par = 0u, v_par = 0u;  // bit i: parity of slot i's next K / V load
  uint32_t last_bar[KVS], last_par[KVS];
#pragma unroll
  for (int i = 0; i < KVS; ++i) last_bar[i] = 0u, last_par[i] = 0u;
  // one K or V tile into the next ring slot
  auto load_kv = [&](const CUtensorMap* map, int row0, const TileInfo& ti, bool is_k) -> bool {
    const int slot = kv_count % KVS, use = kv_count / KVS;
    if (use > 0 && !wait_phase(bars + 8 * (C::B_KV_EMPTY + slot), (use - 1) & 1, abort_flag,
                               p.wait_limit_ns, (kRoleProducer << 8) | kSiteKvEmpty))
      return false;
    const uint32_t full = bars + 8 * ((is_k ? C::B_K_FULL : C::B_V_FULL) + slot);
    uint32_t& par = is_k ? k_par : v_par;
    last_bar[slot] = full;
    last_par[slot] = (par >> slot) & 1u;
    par ^= 1u << slot;
    mbar_arrive_expect_tx(full, C::TILE_BYTES);
#pragma unroll
    for (int c = 0; c < C::CHUNKS; ++c)
      tma_load_4d(base + C::SKV_OFF + slot * C::TILE_BYTES + c * C::CHUNK_BYTES, map, full,
                  c * C::BOX, ti.row0 + row0, ti.h, ti.bc);
    ++kv_count;
    return true;
  };
  // A ring position that carries O instead of a load: once the slot's previous
  // use is released, complete its full phase without bytes, which hands the
  // slot to the softmax groups of the tile (and keeps every slot's phases
  // one per position).
  auto reserve_slot = [&]() -> bool {
    const int slot = kv_count % KVS, use = kv_count / KVS;
    if (use > 0 && !wait_phase(bars + 8 * (C::B_KV_EMPTY + slot), (use - 1) & 1, abort_flag,
                               p.wait_limit_ns, (kRoleProducer << 8) | kSiteKvEmpty))
      return false;
    mbar_arrive(bars + 8 * (C::B_O_READY + slot));
    ++kv_count;
    return true;
  };
  for (int round = 0; ok && round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    if (ti.n_u == 0) continue;
    // The first K tile needs only a ring slot: request it before waiting for
    // the previous work tile to release the Q buffer, so the two loads overlap.
    if (!(ok = load_kv(&p.tmap_k, ti.lo_u * BN, ti, true))) break;
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
                    bars + 8 * C::B_Q_FULL, c * C::BOX, ti.row0 + ti.q0 + s * BM, ti.h, ti.bc);
    ++q_count;
    for (int jj = 0; ok && jj < ti.n_u; ++jj) {
      const int j = ti.lo_u + jj;
      if (jj + 1 < ti.n_u && !(ok = load_kv(&p.tmap_k, (j + 1) * BN, ti, true))) break;
      ok = load_kv(&p.tmap_v, j * BN, ti, false);
    }
#pragma unroll 1
    for (int s = 0; ok && s < QS; ++s)
      if (o_via_slot<C::O_TMA>(p, ti, s)) ok = reserve_slot();
  }
  if (!ok) {
    // Let the loads already issued land before the CTA's shared memory goes away.
    const unsigned long long drain = 10000000ull;
    volatile int no_abort_q = 0;
    if (q_count > 0)
      wait_phase(bars + 8 * C::B_Q_FULL, (q_count - 1) & 1, &no_abort_q, drain,
                 (kRoleProducer << 8) | kSiteDrain);
    // earlier loads into a slot landed before the slot was reused
#pragma unroll 1
    for (int i = 0; i < KVS; ++i) {
      volatile int no_abort = 0;
      if (last_bar[i] != 0u && !mbar_try_wait(last_bar[i], last_par[i]))
        wait_phase(last_bar[i], last_par[i], &no_abort, drain, (kRoleProducer << 8) | kSiteDrain);
    }
  }
}

// The tensor core is fed by two threads, because a thread that issues
// tcgen05.mma runs only about one instruction ahead of its execution: one
// thread issues the S = Q K^T products, the other the O += P V products, so
// that neither waits behind the other's dependencies.  Each commits only what
// it issued.

// S thread, per work tile: S_s(0) for every Q tile s, then S_s(j+1) once the
// softmax of tile s has read S_s(j) out of TMEM.
template <int HD, int QS, int KVS, int ELT>
__device__ void mma_s_role(const FwdParams& p, uint32_t base, uint32_t tmem,
                           volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, ELT>;
  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t idesc_qk =
      ELT == kE4M3 ? e4m3_idesc(BM, BN, false) : f16_idesc(ELT == kBF16, BM, BN, false);
  const unsigned long long lim = p.wait_limit_ns;
  const int G = gridDim.x, cta = blockIdx.x;
  int kv_count = 0, q_count = 0;
  uint32_t sf_par[2] = {0u, 0u};
  int s_issued[2] = {0, 0};
  bool ok = true;

  uint32_t k_par = 0u;  // bit i: parity of slot i's next K load
  auto wait_kv = [&](int idx) -> bool {
    const int slot = idx % KVS;
    const bool r = wait_phase(bars + 8 * (C::B_K_FULL + slot), (k_par >> slot) & 1u, abort_flag,
                              lim, (kRoleMma << 8) | kSiteKvFull);
    k_par ^= 1u << slot;
    tc_fence_after_sync();
    return r;
  };
  // S_s = Q_s K^T into the tile's S buffer, after the softmax has read the
  // buffer's previous contents.  Descriptors are formed once per operand;
  // the K-steps add constant offsets to the low word.
  auto issue_s = [&](int s, int kslot) -> bool {
    if (s_issued[s] > 0) {
      if (!wait_phase(bars + 8 * (C::B_S_FREE + s), sf_par[s], abort_flag, lim,
                      (kRoleMma << 8) | kSiteSFree))
        return false;
      sf_par[s] ^= 1u;
      tc_fence_after_sync();
    }
    const uint32_t qa = sw128_desc_lo(base + C::SQ_OFF + s * C::TILE_BYTES, 16);
    const uint32_t kb = sw128_desc_lo(base + C::SKV_OFF + kslot * C::TILE_BYTES, 16);
    const uint32_t d_tmem = tmem + C::s_col(s);
#pragma unroll
    for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
      const uint32_t off = ((kk / 4) * C::CHUNK_BYTES + (kk % 4) * 32) >> 4;
      if constexpr (ELT == kE4M3)
        mma_ss_f8(d_tmem, desc_from_lo(qa + off), desc_from_lo(kb + off), idesc_qk, kk > 0 ? 1u : 0u);
      else
        mma_ss(d_tmem, desc_from_lo(qa + off), desc_from_lo(kb + off), idesc_qk, kk > 0 ? 1u : 0u);
    }
    tc_commit(bars + 8 * (C::B_S_FULL + s));
    ++s_issued[s];
    return true;
  };

  for (int round = 0; ok && round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    if (ti.n_u == 0) continue;
    ok = wait_phase(bars + 8 * C::B_Q_FULL, q_count & 1, abort_flag, lim,
                    (kRoleMma << 8) | kSiteQFull);
    tc_fence_after_sync();
    ++q_count;
    if (!ok) break;
    const int kv0 = kv_count;
    for (int jj = 0; ok && jj < ti.n_u; ++jj) {
      const int j = ti.lo_u + jj;
      const int k_idx = kv0 + ring_k(jj);
      if (!(ok = wait_kv(k_idx))) break;
#pragma unroll 1
      for (int s = 0; s < QS; ++s)
        if (ok && in_range(ti, s, j)) ok = issue_s(s, k_idx % KVS);
      if (!ok) break;
      tc_commit(bars + 8 * (C::B_KV_EMPTY + k_idx % KVS));
      if (jj + 1 == ti.n_u) tc_commit(bars + 8 * C::B_Q_EMPTY);
    }
    kv_count = kv0 + 2 * ti.n_u + o_slots<C::O_TMA>(p, ti);
  }
  if (!ok) {
    // Wait for every MMA this thread issued before TMEM is released.
    volatile int no_abort = 0;
    tc_commit(bars + 8 * C::B_DRAIN);
    wait_phase(bars + 8 * C::B_DRAIN, 0, &no_abort, 10000000ull, (kRoleMma << 8) | kSiteDrain);
  }
}

// P V thread, per work tile and key block j: O_s (+)= P_s(j) V(j) for tile 0
// then tile 1, each once the softmax has written P_s(j) into the shared P
// buffer; after each product the buffer is handed to the tile that uses it
// next (which also tells that tile's softmax that O_s holds the product).
template <int HD, int QS, int KVS, int ELT>
__device__ void mma_pv_role(const FwdParams& p, uint32_t base, uint32_t tmem,
                            volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, ELT>;
  const uint32_t bars = base + C::BAR_OFF;
  const uint32_t idesc_pv =
      ELT == kE4M3 ? e4m3_idesc(BM, HD, true) : f16_idesc(ELT == kBF16, BM, HD, true);
  const unsigned long long lim = p.wait_limit_ns;
  const int G = gridDim.x, cta = blockIdx.x;
  int kv_count = 0;
  uint32_t p_par = 0u, v_par = 0u;  // v_par bit i: parity of slot i's next V load
  bool ok = true;
  const uint32_t pa = sw128_desc_lo(base + C::SP_OFF, 16);

  // O (+)= P V with P read from shared memory, handed over in two halves of
  // 64 keys: the first four K-steps start once the first half is written and
  // both halves of O are rescaled.  Once a half's K-steps have run, that half
  // of the buffer goes to the next user (tile `nxt`).
  auto issue_pv = [&](int s, int vslot, bool accumulate, int nxt) -> bool {
    const uint32_t vb = sw128_desc_lo(base + C::SKV_OFF + vslot * C::TILE_BYTES, C::CHUNK_BYTES);
    const uint32_t d_tmem = tmem + (s ? C::O_COL1 : C::O_COL0);
    // Byte offset of the first key of half h in a P row: 64 keys of 16 bits
    // fill one 128-byte chunk, 64 e4m3 keys half of one.
    constexpr int HALF_STEPS = C::PV_KSTEPS / 2;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (!wait_phase(bars + 8 * (C::B_P_FULL + half), p_par, abort_flag, lim,
                      (kRoleMma << 8) | kSitePFull))
        return false;
      tc_fence_after_sync();
      const int half_off = C::EB == 2 ? half * C::CHUNK_BYTES : half * 64;
#pragma unroll
      for (int k = 0; k < HALF_STEPS; ++k) {
        const int kk = half * HALF_STEPS + k;
        const uint64_t a = desc_from_lo(pa + ((half_off + k * 32) >> 4));
        const uint64_t b = desc_from_lo(vb + ((kk * C::KSTEP * 128) >> 4));
        if constexpr (ELT == kE4M3)
          mma_ss_f8(d_tmem, a, b, idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
        else
          mma_ss(d_tmem, a, b, idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
      }
      tc_commit(bars + 8 * (C::B_P_FREE + 2 * nxt + half));
    }
    tc_commit(bars + 8 * (C::B_PV_DONE + s));
    p_par ^= 1u;
    return true;
  };

  for (int round = 0; ok && round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    if (ti.n_u == 0) continue;
    const int kv0 = kv_count;
    for (int jj = 0; ok && jj < ti.n_u; ++jj) {
      const int j = ti.lo_u + jj;
      const int v_idx = kv0 + ring_v(jj, ti.n_u);
      ok = wait_phase(bars + 8 * (C::B_V_FULL + v_idx % KVS), (v_par >> (v_idx % KVS)) & 1u,
                      abort_flag, lim, (kRoleMma << 8) | kSiteKvFull);
      v_par ^= 1u << (v_idx % KVS);
      tc_fence_after_sync();
#pragma unroll 1
      for (int s = 0; s < QS; ++s) {
        if (!ok || !in_range(ti, s, j)) continue;
        // the next work tile starts with tile 0
        const int nxt = next_p_user(s, j, ti);
        ok = issue_pv(s, v_idx % KVS, j > ti.lo[s], nxt < 0 ? 0 : nxt);
        if (!ok) break;
        if (j == ti.hi[s] - 1) tc_commit(bars + 8 * (C::B_O_FINAL + s));
      }
      if (!ok) break;
      tc_commit(bars + 8 * (C::B_KV_EMPTY + v_idx % KVS));
    }
    kv_count = kv0 + 2 * ti.n_u + o_slots<C::O_TMA>(p, ti);
  }
  if (!ok) {
    volatile int no_abort = 0;
    tc_commit(bars + 8 * (C::B_DRAIN + 1));
    wait_phase(bars + 8 * (C::B_DRAIN + 1), 0, &no_abort, 10000000ull,
               (kRoleMma << 8) | kSiteDrain);
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

// Max of 64 scores as a balanced tree of 3-input maxima.
__device__ __forceinline__ float row_max64(const float* sv) {
  float t[22];
#pragma unroll
  for (int i = 0; i < 21; ++i) t[i] = max3(sv[3 * i], sv[3 * i + 1], sv[3 * i + 2]);
  t[21] = sv[63];
  float u[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) u[i] = max3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
  u[7] = t[21];
  return fmaxf(max3(u[0], u[1], u[2]), max3(u[3], u[4], fmaxf(u[5], fmaxf(u[6], u[7]))));
}

// Writes 64 keys of one P row (32 packed pairs) into the 128-byte swizzled,
// K-major layout the P V MMA reads: row r of a 64-key chunk at r * 128 bytes,
// its 16-byte group u at position u ^ (r % 8).
__device__ __forceinline__ void store_p_chunk(uint32_t chunk_base, int r, const uint32_t* pk) {
  const uint32_t row = chunk_base + static_cast<uint32_t>(r) * 128u;
#pragma unroll
  for (int u = 0; u < 8; ++u)
    st_shared_v4(row + ((static_cast<uint32_t>(u) ^ (r & 7u)) << 4), pk[4 * u], pk[4 * u + 1],
                 pk[4 * u + 2], pk[4 * u + 3]);
}

// Exponentials, row-sum and 16-bit packing of 32 consecutive scores.
// POLY8 of every 8 argument pairs go through exp2_poly2, the rest through ex2.
// The row sum goes into four independent packed accumulators, so the adds
// form four short dependency chains instead of one long one.
// 16-bit P: pk[q] holds keys 2q, 2q+1.  e4m3 P: pk[q / 2] holds keys
// 4(q/2) .. 4(q/2)+3, low byte first (so pk covers 16 words, not 32).
template <int ELT, int POLY8>
__device__ __forceinline__ void softmax_chunk(const float* sv, float sl2, float neg_ref,
                                              uint32_t* pk, float2 (&acc)[4]) {
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
    acc[q & 3] = __fadd2_rn(acc[q & 3], e);
    if constexpr (ELT == kE4M3) {
      const uint32_t h = pack_e4m3x2(e.x, e.y);
      if (q & 1)
        pk[q / 2] |= h << 16;
      else
        pk[q / 2] = h;
    } else {
      pk[q] = pack2<ELT == kBF16>(e.x, e.y);
    }
  }
}

// Writes 64 e4m3 keys of one P row (16 words) into its half (bytes 64 hf ..
// 64 hf + 63) of the row's 128-byte swizzled line: 16-byte group u of the
// line at position u ^ (r % 8).
__device__ __forceinline__ void store_p_half_e4m3(uint32_t p_base, int r, int hf,
                                                  const uint32_t* pk) {
  const uint32_t row = p_base + static_cast<uint32_t>(r) * 128u;
#pragma unroll
  for (int u = 0; u < 4; ++u)
    st_shared_v4(row + ((static_cast<uint32_t>(4 * hf + u) ^ (r & 7u)) << 4), pk[4 * u],
                 pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
}

// ALIBI: the scaled score of key j gets -slope[h] * |i - j| (in the log2
// domain, -slope[h] * log2(e) * |i - j|) before the row max is taken.
template <int HD, int QS, int KVS, int ELT, bool ALIBI>
__device__ void softmax_role(const FwdParams& p, uint32_t base, uint32_t tmem,
                             volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, ELT>;
  constexpr bool OUT_BF16 = ELT != kF16;  // e4m3 inputs give a bf16 output
  using T = typename std::conditional<OUT_BF16, __nv_bfloat16, __half>::type;
  constexpr int HD2 = HD / 2;                 // O columns each group of a tile owns
  const uint32_t bars = base + C::BAR_OFF;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int wg = warp / 4;
  const int s = wg >> 1;                      // which Q tile of the work tile
  const int hf = wg & 1;                      // which 64 key columns of its S rows
  const int r = (warp % 4) * 32 + lane;       // query row within the tile == TMEM lane
  const uint32_t lane_base = tmem + ((static_cast<uint32_t>(warp % 4) * 32u) << 16);
  const uint32_t s_col = C::s_col(s) + 64u * hf;
  const uint32_t o_col = (s ? C::O_COL1 : C::O_COL0) + HD2 * hf;
  // this group's half of P: its own chunk (16-bit), or half of each line (e4m3)
  const uint32_t sp = base + C::SP_OFF + (C::EB == 2 ? hf * C::CHUNK_BYTES : 0);
  float* xch = reinterpret_cast<float*>(
      __cvta_shared_to_generic(base + C::XCH_OFF));
  float* x_mine = xch + (s * 2 + hf) * 128;
  const float* x_other = xch + (s * 2 + (hf ^ 1)) * 128;
  const unsigned long long lim = p.wait_limit_ns;
  const float sl2 = p.scale_log2;
  const int G = gridDim.x, cta = blockIdx.x;
  uint32_t s_par = 0u, pf_par = 0u, fin_par = 0u, x_par = 0u;
  int pv_count = 0;  // P V products of this Q tile issued before the current block
  int kv_count = 0;  // ring positions of the work tiles so far (for the O slots)
  uint32_t o_par = 0u;  // bit i: parity of slot i's next O reservation (both tiles' O)
  // The P buffer's first use in the kernel (tile 0, first block) has nothing
  // to wait for; every later use waits for the buffer to be handed over.
  bool first_use = s == 0;
  // Both softmax groups of the tile arrive (one arrival per warp, after the
  // warp's shared-memory writes) and wait for each other, with the bounded wait.
  auto group_meet = [&]() -> bool {
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + 8 * (C::B_XCH + s));
    const bool met = wait_phase(bars + 8 * (C::B_XCH + s), x_par, abort_flag, lim,
                                (kRoleSoftmax << 8) | kSiteXch);
    x_par ^= 1u;
    return __all_sync(0xffffffffu, met);
  };

  for (int round = 0; round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    // ring slot of this tile's O and the parity of its reservation; every
    // group follows the reservations of both tiles
    int o_slot = -1;
    uint32_t o_wait_par = 0u;
    if (ti.n_u > 0) {
      int k = 0;
#pragma unroll 1
      for (int s2 = 0; s2 < QS; ++s2) {
        if (!o_via_slot<C::O_TMA>(p, ti, s2)) continue;
        const int slot = (kv_count + 2 * ti.n_u + k++) % KVS;
        if (s2 == s) {
          o_slot = slot;
          o_wait_par = (o_par >> slot) & 1u;
        }
        o_par ^= 1u << slot;
      }
      kv_count += 2 * ti.n_u + k;
    }
    const int lo = ti.lo[s], hi = ti.hi[s];
    if (lo == hi) continue;
    const int r_first = ti.q0 + s * BM, r_last = r_first + BM - 1;
    const int row = r_first + r;  // relative to the sequence
    // keys visible from this row: [vis_lo, vis_hi)
    const int vis_lo = p.window_left < 0 ? 0 : row - p.window_left;
    const int vis_hi = p.window_right < 0 ? ti.len : min(ti.len, row + p.window_right + 1);
    float nslope2 = 0.f;  // -slope * log2(e)
    if constexpr (ALIBI) nslope2 = -__ldg(p.alibi_slopes + ti.h) * 1.4426950408889634f;
    float m_ref = -INFINITY, l = 0.f;

    for (int j = lo; j < hi; ++j) {
      bool ok = wait_phase(bars + 8 * (C::B_S_FULL + s), s_par, abort_flag, lim,
                           (kRoleSoftmax << 8) | kSiteSFull);
      s_par ^= 1u;
      if (!__all_sync(0xffffffffu, ok)) return;
      tc_fence_after_sync();
      uint32_t sr[64];
      tmem_ld64_nowait(lane_base + s_col, sr);
      tmem_ld64_wait(sr);
      float sv[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) sv[c] = __uint_as_float(sr[c]);
      // Blocks where some key is invisible to some row of the tile: the ragged
      // tail, the causal diagonal, the edges of a local window.
      const bool need_mask =
          (j * BN + BN > ti.len) ||
          (p.window_left >= 0 && j * BN < r_last - p.window_left) ||
          (p.window_right >= 0 && j * BN + BN - 1 > r_first + p.window_right);
      const int kbase = j * BN + 64 * hf;  // key of this thread's first column
      if (need_mask) {
        const int lo_c = vis_lo - kbase, hi_c = vis_hi - kbase;
#pragma unroll
        for (int c = 0; c < 64; ++c) sv[c] = (c >= lo_c && c < hi_c) ? sv[c] : -INFINITY;
      }
      float m_half;
      if constexpr (ALIBI) {
        // log2-domain biased scores; the max is taken over them
        const float dist0 = static_cast<float>(row - kbase);
#pragma unroll
        for (int c = 0; c < 64; ++c)
          sv[c] = fmaf(sv[c], sl2, nslope2 * fabsf(dist0 - static_cast<float>(c)));
        m_half = row_max64(sv);
      } else {
        // row max over both halves of the row
        m_half = row_max64(sv) * sl2;
      }
      x_mine[r] = m_half;
      if (!group_meet()) return;
      const float m_blk = fmaxf(m_half, x_other[r]);
      // S is in registers and both groups have read the exchange slot: the S
      // thread may overwrite the S buffer with S(j+1), and the slots are free
      // again once that S arrives.
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (C::B_S_FREE + s));

      // Lazy reference: keep m_ref unless the block max exceeds it by more
      // than 2^8; the first block always sets it.  Both groups of the tile
      // take the same decision from the same values.
      // A row with no visible key so far (m_ref = -inf: only possible at the
      // edges of a local window) has l = 0 and O = 0, so its alpha is 0.
      const bool rescale = (j > lo) && (m_blk > m_ref + kLazyRescaleLog2);
      const float m_new = (j == lo || rescale) ? m_blk : m_ref;
      const float alpha =
          (j == lo || m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);  // 1 when m_ref is kept
      m_ref = m_new;
      const float neg_ref = (m_ref == -INFINITY) ? 0.f : -m_ref;
      const float sl2e = ALIBI ? 1.f : sl2;  // the ALiBi path holds scaled scores already

      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
      constexpr int PK_WORDS = 32 * C::EB / 2;  // words of P per 32 keys, times 2
      uint32_t pk[PK_WORDS];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (need_mask)
          softmax_chunk<ELT, 0>(sv + 32 * c, sl2e, neg_ref, pk + (PK_WORDS / 2) * c, acc);
        else
          softmax_chunk<ELT, poly_pairs_per8<HD>()>(sv + 32 * c, sl2e, neg_ref,
                                                    pk + (PK_WORDS / 2) * c, acc);
      }
      // This group's half of the P buffer is this tile's turn: the previous
      // user's K-steps that read it have run.
      if (!first_use) {
        ok = wait_phase(bars + 8 * (C::B_P_FREE + 2 * s + hf), pf_par, abort_flag, lim,
                        (kRoleSoftmax << 8) | kSitePFree);
        pf_par ^= 1u;
        if (!__all_sync(0xffffffffu, ok)) return;
        tc_fence_after_sync();
      }
      first_use = false;
      if (__any_sync(0xffffffffu, rescale)) {
        // O must hold P V_s(j-1) before it is rescaled.  Every earlier product
        // of the tile is known to have finished (the buffer hand-overs came
        // after them) and the next one needs this block's P, so the phase of
        // P V_s(j-1) is the barrier's current or just completed one.
        ok = wait_phase(bars + 8 * (C::B_PV_DONE + s), static_cast<uint32_t>(pv_count - 1) & 1u,
                        abort_flag, lim, (kRoleSoftmax << 8) | kSitePFree);
        if (!__all_sync(0xffffffffu, ok)) return;
        tc_fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < HD2; c += 16) {
          uint32_t ov[16];
          tmem_ld16_sync(lane_base + o_col + c, ov);
#pragma unroll
          for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st16(lane_base + o_col + c, ov);
        }
        tmem_st_wait();
      }
      // The first P V K-steps write all of O: the second group reports its
      // half rescaled on the barrier of the first P half.
      if (hf == 1) {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * C::B_P_FULL);
      }
      if constexpr (ELT == kE4M3)
        store_p_half_e4m3(sp, r, hf, pk);
      else
        store_p_chunk(sp, r, pk);
      // make the generic-proxy stores visible to the tensor core
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (C::B_P_FULL + hf));
      ++pv_count;
      const float2 acc01 = __fadd2_rn(acc[0], acc[1]), acc23 = __fadd2_rn(acc[2], acc[3]);
      l = l * alpha + ((acc01.x + acc23.x) + (acc01.y + acc23.y));
    }

    // Epilogue: wait for the last P V product; each group writes its half of
    // the O columns, divided by the row sum of both halves.
    bool ok = wait_phase(bars + 8 * (C::B_O_FINAL + s), fin_par, abort_flag, lim,
                         (kRoleSoftmax << 8) | kSiteODone);
    fin_par ^= 1u;
    if (!__all_sync(0xffffffffu, ok)) return;
    tc_fence_after_sync();
    x_mine[r] = l;
    if (!group_meet()) return;
    const float l_row = l + x_other[r];
    if (!group_meet()) return;  // both have read before the slots are reused
    const float inv_l = p.o_scale / l_row;
    const long long trow = static_cast<long long>(ti.row0) + row;  // tensor row
    const bool store = row < ti.len && trow < p.rows_total;
    if (o_slot >= 0) {
      // Stage this group's columns of O in the tile's ring slot, in the
      // 128-byte swizzled layout of the TMA box (row r's 16-byte unit u at
      // u ^ (r % 8) of its line), for the store warp to write out by TMA.
      const int slot = o_slot;
      bool ok = wait_phase(bars + 8 * (C::B_O_READY + slot), o_wait_par, abort_flag, lim,
                           (kRoleSoftmax << 8) | kSiteOSlot);
      if (!__all_sync(0xffffffffu, ok)) return;
      const uint32_t sbase = base + C::SKV_OFF + slot * C::TILE_BYTES + r * 128;
#pragma unroll 1
      for (int c = 0; c < HD2; c += 32) {
        uint32_t ov[32];
        tmem_ld32_sync(lane_base + o_col + c, ov);
        uint32_t wp[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wp[i] = pack2<OUT_BF16>(__uint_as_float(ov[2 * i]) * inv_l,
                                  __uint_as_float(ov[2 * i + 1]) * inv_l);
        const int col = HD2 * hf + c;  // first of these 32 columns
        const uint32_t line = sbase + (col / 64) * C::CHUNK_BYTES;
        const uint32_t u0 = (col % 64) / 8;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          st_shared_v4(line + (((u0 + i) ^ (static_cast<uint32_t>(r) & 7u)) << 4), wp[4 * i],
                       wp[4 * i + 1], wp[4 * i + 2], wp[4 * i + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (C::B_O_STAGED + slot));
    } else {
    T* orow = reinterpret_cast<T*>(p.o) + ti.bc * p.o_stride_b + ti.h * p.o_stride_h +
              trow * p.o_stride_n + HD2 * hf;
#pragma unroll 1
    for (int c = 0; c < HD2; c += 32) {
      uint32_t ov[32];
      tmem_ld32_sync(lane_base + o_col + c, ov);
      uint4 w[4];
      uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        wp[i] = pack2<OUT_BF16>(__uint_as_float(ov[2 * i]) * inv_l,
                                __uint_as_float(ov[2 * i + 1]) * inv_l);
      if (store) {
        if (p.o_vec32) {
          // 32-byte stores: every store fills whole 32-byte sectors
          st_global_v8(orow + c, wp);
          st_global_v8(orow + c + 16, wp + 8);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = w[i];
        }
      }
    }
    }
    if (hf == 0 && p.lse != nullptr && store)
      p.lse[ti.bc * p.lse_stride_b + ti.h * p.lse_stride_h + trow] =
          (m_ref + log2f(l_row)) * 0.69314718055994530942f;
    // The next tile's first P V overwrites O only after this group's next
    // P arrival, which comes after these loads completed.
    tc_fence_before_sync();
  }
}

// Store warp (one thread): for every Q tile whose O goes through a ring slot,
// waits until both softmax groups have staged their columns there, writes the
// tile out with TMA stores, waits until the stores have read the slot and
// releases it to the producer.
template <int HD, int QS, int KVS, int ELT>
__device__ void store_role(const FwdParams& p, uint32_t base, volatile int* abort_flag) {
  using C = FwdCfg<HD, QS, KVS, ELT>;
  const uint32_t bars = base + C::BAR_OFF;
  const int G = gridDim.x, cta = blockIdx.x;
  int kv_count = 0;
  uint32_t staged_par = 0u;  // bit i: parity of ring slot i's next staging
  bool ok = true;
  for (int round = 0; ok && round * G < p.num_tiles; ++round) {
    const int t = tile_of(round, cta, G);
    if (t >= p.num_tiles) continue;
    const TileInfo ti = decode_tile<QS>(p, t);
    if (ti.n_u == 0) continue;
    const int kv0 = kv_count;
    kv_count += 2 * ti.n_u + o_slots<C::O_TMA>(p, ti);
    int k = 0;
#pragma unroll 1
    for (int s = 0; s < QS; ++s) {
      if (!o_via_slot<C::O_TMA>(p, ti, s)) continue;
      const int slot = (kv0 + 2 * ti.n_u + k++) % KVS;
      ok = wait_phase(bars + 8 * (C::B_O_STAGED + slot), (staged_par >> slot) & 1u, abort_flag,
                      p.wait_limit_ns, (kRoleStore << 8) | kSiteOStaged);
      staged_par ^= 1u << slot;
      if (!ok) break;
      const uint32_t src = base + C::SKV_OFF + slot * C::TILE_BYTES;
#pragma unroll
      for (int c = 0; c < C::CHUNKS; ++c)
        tma_store_4d(&p.tmap_o, src + c * C::CHUNK_BYTES, c * C::BOX, ti.row0 + ti.q0 + s * BM,
                     ti.h, ti.bc);
      bulk_commit_group();
      bulk_wait_read_all();
      mbar_arrive(bars + 8 * (C::B_KV_EMPTY + slot));
    }
  }
  // the writes themselves complete before the CTA ends
  bulk_wait_all();
}

template <int HD, int QS, int KVS, int ELT, bool ALIBI>
__global__ void __launch_bounds__(FwdCfg<HD, QS, KVS, ELT>::THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<HD, QS, KVS, ELT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  if (base - raw > static_cast<uint32_t>(C::ALIGN_SLACK)) {
    // the 1024-byte-aligned layout would not fit the allocation: refuse
    if (threadIdx.x == 0) atomicCAS(&g_fa_watchdog, 0u, (kRoleTest << 8) | kSiteAlign);
    return;
  }
  uint8_t* smem = smem_raw + (base - raw);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  const uint32_t bars = base + C::BAR_OFF;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(bars + 8 * C::B_Q_FULL, 1);
    mbar_init(bars + 8 * C::B_Q_EMPTY, 1);
    for (int i = 0; i < KVS; ++i) {
      mbar_init(bars + 8 * (C::B_K_FULL + i), 1);
      mbar_init(bars + 8 * (C::B_V_FULL + i), 1);
      mbar_init(bars + 8 * (C::B_O_READY + i), 1);
      mbar_init(bars + 8 * (C::B_KV_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars + 8 * (C::B_XCH + i), 8);  // one arrival per softmax warp of the tile
      mbar_init(bars + 8 * (C::B_S_FULL + i), 1);
      mbar_init(bars + 8 * (C::B_S_FREE + i), 8);  // one arrival per softmax warp of the tile
      mbar_init(bars + 8 * (C::B_P_FREE + 2 * i), 1);
      mbar_init(bars + 8 * (C::B_P_FREE + 2 * i + 1), 1);
      mbar_init(bars + 8 * (C::B_PV_DONE + i), 1);
      mbar_init(bars + 8 * (C::B_O_FINAL + i), 1);
      mbar_init(bars + 8 * (C::B_DRAIN + i), 1);
    }
    for (int i = 0; i < KVS; ++i)
      mbar_init(bars + 8 * (C::B_O_STAGED + i), 8);  // one arrival per softmax warp of the tile
    // first P half: the first group's warps once P is written and the second
    // group's once their O half is rescaled; second half: the second group
    mbar_init(bars + 8 * C::B_P_FULL, 8);
    mbar_init(bars + 8 * (C::B_P_FULL + 1), 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    tma_prefetch_desc(&p.tmap_q);
    tma_prefetch_desc(&p.tmap_k);
    tma_prefetch_desc(&p.tmap_v);
    if (C::O_TMA) tma_prefetch_desc(&p.tmap_o);
  }
  if (warp == C::MMA_S_WARP) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if constexpr (C::REG_SPLIT) {
    if (warp < C::SOFTMAX_WARPS)
      reg_alloc<C::SOFTMAX_REGS>();
    else
      reg_dealloc<C::OTHER_REGS>();
  }

  if (warp < C::SOFTMAX_WARPS) {
    softmax_role<HD, QS, KVS, ELT, ALIBI>(p, base, tmem, abort_flag);
  } else if (warp == C::PRODUCER_WARP) {
    if (lane == 0) producer_role<HD, QS, KVS, ELT>(p, base, abort_flag);
  } else if (warp == C::MMA_S_WARP) {
    if (lane == 0) mma_s_role<HD, QS, KVS, ELT>(p, base, tmem, abort_flag);
  } else if (warp == C::MMA_PV_WARP) {
    if (lane == 0) mma_pv_role<HD, QS, KVS, ELT>(p, base, tmem, abort_flag);
  } else if (warp == C::STORE_WARP) {
    if (lane == 0 && C::O_TMA) store_role<HD, QS, KVS, ELT>(p, base, abort_flag);
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == C::MMA_S_WARP) {
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
