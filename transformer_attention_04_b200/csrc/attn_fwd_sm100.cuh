// Fused RoPE + grouped-query causal attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes: out = softmax(Q' K'^T / sqrt(D) + M) V per (batch, query head), where
// Q' and K' are the RoPE-rotated queries and keys, M is -inf above the causal diagonal,
// and query head h reads key/value head h / (Hq/Hkv). This is the scaled dot-product
// attention of "Multi-Head Attention & Rotary Position Embeddings (RoPE)" (learnllm.online,
// "Scaled Dot-Product Attention: The O(S^2) Memory Wall") with the grouped-query sharing of
// "Transformer internals: attention without the mysticism" (ninaddeshpande.com, "The KV
// cache and the memory wall"). The [B,H,S,S] scores never reach HBM: they are produced
// tile by tile in tensor memory and folded with the online softmax (running row max and
// row sum, rescaling the partial output) that "Transformer Architecture & Self-Attention
// Mechanics" (devthesis.com, §4 "The Quadratic Bottleneck & FlashAttention") and
// "Transformer Architecture: FlashAttention & RoPE" (KWAS Academy, "Line-by-Line
// Technical Breakdown") describe.
//
// One CTA = one work unit = up to two 128-row query tiles ("slots") that share every K/V
// tile: two query heads of the same KV group at the same positions (GQA with an even group
// size) or, for odd group sizes, a single tile. Warp roles (384 threads):
//   warp 0        TMA producer: Q tiles once, then K'/V tiles into an NST-deep ring.
//   warp 1        TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 2-3     idle.
//   warps 4-7     softmax warpgroup of slot 0 (thread = query row = TMEM lane).
//   warps 8-11    softmax warpgroup of slot 1.
// Per KV tile j the issuer runs S_s = Q_s K_j^T (SS MMA, fp32 in TMEM), the softmax
// group turns S_s into bf16 P_s written over the same TMEM columns, and the issuer runs
// O_s += P_s V_j with P taken from TMEM (TS MMA). Issue order S0 S1 | PV0 S0' PV1 S1' ...
// keeps one slot's softmax overlapping the other slot's MMAs. tcgen05.mma issued by one
// thread execute in order, so S_s(j+1) never overwrites P_s(j) before PV_s(j) has read it,
// and each commit after S_s(j) also covers PV_s(j-1) (used before rescaling O_s).
//
// Q is rotated in shared memory by its softmax group right after the TMA load; K is
// rotated once per call by rope_rotate_kernel into a workspace, since every K tile is
// re-read by S/128 query tiles.
#pragma once

#include "ptx.cuh"
#include "rope.cuh"

namespace ra {

#ifdef RA_TRACE
// Per-phase clock64() stamps of CTAs 0-1 for the first 64 KV tiles (profiling builds only).
__device__ unsigned long long g_trace[2][16][64];
#define RA_STAMP(ev, j)                                                         \
  do {                                                                          \
    if (blockIdx.x < 2 && (j) < 64) g_trace[blockIdx.x][(ev)][(j)] = clock64(); \
  } while (0)
#else
#define RA_STAMP(ev, j) \
  do {                  \
  } while (0)
#endif

constexpr float kLn2 = 0.6931471805599453f;

struct FwdParams {
  __nv_bfloat16* out;   // [B, Hq, Sq, D]
  const float2* tab;    // RoPE (cos, sin) table, D/2 entries per position
  unsigned int* status; // sticky device status word
  long long wait_limit; // polls per mbarrier wait before giving up
  int B, Hq, Hkv, Sq, Sk;
  int G;                // Hq / Hkv
  int n_slots;          // query tiles per CTA (1 or 2)
  int ppg;              // CTA units per (batch, KV group, query tile) = G / n_slots
  int n_qtiles;         // ceil(Sq / 128)
  int causal;
  int off;              // query row i sits at key index i + off (causal: key j allowed iff j <= i + off)
  int window;           // 0 = none; else key j is allowed to query row i iff j > i + off - window
  int q_tab_off;        // table row of query row 0
  float scale_log2;     // log2(e) / sqrt(D)
  // partial (ring) mode when o_acc is set: O / l in fp32 [B, Hq, Sq, D] and the row's natural
  // log-sum-exp in lse_acc [B, Hq, Sq], merged into their contents when accumulate is set;
  // `out` (bf16) is then optional and receives the merged result
  float* o_acc;
  float* lse_acc;
  int accumulate;
  int acc_rows;  // partial mode: rows between heads in o_acc / lse_acc / out (>= Sq)
};

template <int D>
struct FwdCfg {
  static constexpr int KB = D / 64;                  // 128-byte column blocks per row
  static constexpr int BLK = 128 * 128;              // bytes of one 128-row column block
  static constexpr int TILE = 128 * D * 2;           // bytes of one 128 x D bf16 tile
  // K and V tiles stream through one ring in the order K0 V0 K1 V1 ...: 5 slots at D = 128
  // (2.5 KV tiles of look-ahead; 2 Q tiles + 5 slots = 224 KB of shared memory).
  static constexpr int NSLOT = (D == 128) ? 5 : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + 2 * TILE;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * TILE;
  static constexpr int SMEM = OFF_BAR + 512;  // the dynamic shared base is 1024-aligned (checked)
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns: S/P of slot s at 128*s, O of slot s at 256 + D*s
  __device__ static constexpr uint32_t col_s(int s) { return 128u * static_cast<uint32_t>(s); }
  __device__ static constexpr uint32_t col_o(int s) { return 256u + static_cast<uint32_t>(D * s); }
  // barrier indices (8 bytes each)
  static constexpr int B_QFULL = 0, B_QREADY = 2, B_SFULL = 4, B_PFULL = 6, B_OFULL = 8,
                       B_DRAIN = 10, B_FULL = 11, B_EMPTY = 11 + NSLOT, N_BAR = 11 + 2 * NSLOT;
  static constexpr int OFF_TMEM_SLOT = 8 * N_BAR;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
  static_assert(OFF_ABORT + 4 <= 512, "barrier area");
  static_assert(SMEM <= 232448, "shared memory per block");
};

// P = 2^(s * sl2 - m) for one 128-column row of S held in registers; writes the bf16 P
// over the first 64 TMEM columns at tS and returns the row sum of the fp32 values.
// Pairs go through one packed FMA; kEmu of every 4 pairs use the FMA-pipe exponential.
template <int kEmu>
__device__ __forceinline__ float softmax_p_store(const uint32_t* sr, float sl2, float m,
                                                 uint32_t tS) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m, -m);
  uint64_t acc2[4] = {0, 0, 0, 0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int c2 = 0; c2 < 32; ++c2) {
      const int c = h * 64 + 2 * c2;
      const uint64_t x2 =
          f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm2);
      uint64_t p2;
      if ((c2 & 3) < kEmu) {
        p2 = exp2_poly_x2(x2);
      } else {
        float x0, x1;
        f2_unpack(x2, x0, x1);
        p2 = f2_pack(ex2(x0), ex2(x1));
      }
      acc2[c2 & 3] = f2_add(acc2[c2 & 3], p2);
      float p0, p1;
      f2_unpack(p2, p0, p1);
      pk[c2] = pack_bf16(p0, p1);
    }
    tmem_st32(tS + 32 * h, pk);
  }
  const uint64_t a = f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3]));
  float a0, a1;
  f2_unpack(a, a0, a1);
  return a0 + a1;
}

// Same as softmax_p_store, and also returns the max of the 128 raw scores in `mt` (eight
// independent 3-input max chains interleaved with the exponentials, off the critical path).
template <int kEmu>
__device__ __forceinline__ float softmax_p_store_max(const uint32_t* sr, float sl2, float m,
                                                     uint32_t tS, float& mt) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m, -m);
  uint64_t acc2[4] = {0, 0, 0, 0};
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int c2 = 0; c2 < 32; ++c2) {
      const int c = h * 64 + 2 * c2;
      const float s0 = __uint_as_float(sr[c]), s1 = __uint_as_float(sr[c + 1]);
      mx[c2 & 7] = max3f(mx[c2 & 7], s0, s1);
      const uint64_t x2 = f2_fma(f2_pack(s0, s1), sl2x2, negm2);
      uint64_t p2;
      if ((c2 & 3) < kEmu) {
        p2 = exp2_poly_x2(x2);
      } else {
        float x0, x1;
        f2_unpack(x2, x0, x1);
        p2 = f2_pack(ex2(x0), ex2(x1));
      }
      acc2[c2 & 3] = f2_add(acc2[c2 & 3], p2);
      float p0, p1;
      f2_unpack(p2, p0, p1);
      pk[c2] = pack_bf16(p0, p1);
    }
    tmem_st32(tS + 32 * h, pk);
  }
  mt = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
  const uint64_t a = f2_add(f2_add(acc2[0], acc2[1]), f2_add(acc2[2], acc2[3]));
  float a0, a1;
  f2_unpack(a, a0, a1);
  return a0 + a1;
}

#ifndef RA_EMU_PAIRS
#define RA_EMU_PAIRS 0
#endif

// kEmuPairs: of every 4 column pairs of an unmasked tile, how many take the FMA-pipe
// exponential (0 = all on the MUFU).
template <int D, int kEmuPairs = RA_EMU_PAIRS>
__global__ void __launch_bounds__(384, 1)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t base = smem_u32(smem);
  if (base & 1023u) {  // the 128-byte swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.status, kStatusLayout);
    return;
  }
  const uint32_t sQ = base + C::OFF_Q, sRing = base + C::OFF_RING;
  const uint32_t sBar = base + C::OFF_BAR;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_BAR + C::OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_BAR + C::OFF_TMEM_SLOT);
  auto bar = [&](int i) -> uint32_t { return sBar + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit (blockIdx order = longest causal extent first)
  const int per_tile = p.B * p.Hkv * p.ppg;
  const int t_rank = blockIdx.x / per_tile;
  const int rem = blockIdx.x - t_rank * per_tile;
  const int qt = p.causal ? (p.n_qtiles - 1 - t_rank) : t_rank;
  const int b = rem / (p.Hkv * p.ppg);
  const int g = (rem / p.ppg) % p.Hkv;
  const int hp = rem % p.ppg;
  const int h0 = g * p.G + hp * p.n_slots;
  const int kv_bh = b * p.Hkv + g;
  const int q0 = qt * 128;
  const int off = p.off;  // query row i sits at key index i + off
  int n_kv = (p.Sk + 127) / 128;
  if (p.causal) n_kv = min(n_kv, (min(p.Sq - 1, q0 + 127) + off) / 128 + 1);
  // with a sliding window, tiles wholly below the first row's window are skipped too
  const int j_lo = (p.window > 0) ? max(0, q0 + off - p.window + 1) / 128 : 0;
  const int n_it = n_kv - j_lo;  // KV tiles this CTA visits: j_lo .. n_kv - 1
  const int ns = p.n_slots;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::B_QFULL + s), 1);
      mbar_init(bar(C::B_QREADY + s), 4);  // one arrival per softmax warp
      mbar_init(bar(C::B_SFULL + s), 1);
      mbar_init(bar(C::B_PFULL + s), 4);
      mbar_init(bar(C::B_OFULL + s), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(bar(C::B_FULL + i), 1);
      mbar_init(bar(C::B_EMPTY + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Register split: launched at 168 per thread (384 x 168 = 64512); the control
  // warpgroup gives back to 80, the two softmax warpgroups take 208
  // (128 x 80 + 256 x 208 = 63488 <= 64512).
  if (warp < 4) {
  regs_dec<80>();
  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      // K/V tiles are re-read by every query tile of their head group: keep them in L2;
      // each Q tile is read once.
      const uint64_t pol_keep = l2_policy_evict_last();
      const uint64_t pol_once = l2_policy_evict_first();
      for (int s = 0; s < ns; ++s) {
        mbar_expect_tx(bar(C::B_QFULL + s), C::TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d_hint(sQ + s * C::TILE + kb * C::BLK, &tm_q, kb * 64, q0, b * p.Hq + h0 + s,
                           bar(C::B_QFULL + s), pol_once);
      }
      // ring item i: tile i/2 of K (i even) or V (i odd), in slot i % NSLOT
      int issued = 0;
      for (int i = 0; i < 2 * n_it; ++i) {
        const int sl = i % C::NSLOT;
        if (!(i & 1)) RA_STAMP(14, i >> 1);
        if (i >= C::NSLOT && !mbar_wait(bar(C::B_EMPTY + sl), ((i / C::NSLOT) - 1) & 1,
                                        p.wait_limit, abort_flag, p.status))
          break;
        RA_STAMP(12 + (i & 1), i >> 1);
        mbar_expect_tx(bar(C::B_FULL + sl), C::TILE);
        const CUtensorMap* map = (i & 1) ? &tm_v : &tm_k;
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d_hint(sRing + sl * C::TILE + kb * C::BLK, map, kb * 64, (j_lo + (i >> 1)) * 128, kv_bh,
                           bar(C::B_FULL + sl), pol_keep);
        issued = i + 1;
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA can exit
        for (int s = 0; s < ns; ++s) mbar_drain(bar(C::B_QFULL + s), 0);
        for (int i = max(0, issued - C::NSLOT); i < issued; ++i)
          mbar_drain(bar(C::B_FULL + i % C::NSLOT), (i / C::NSLOT) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_bf16(128, 128, 0, 0);  // Q, K both K-major
      constexpr uint32_t kIdescO = umma_idesc_bf16(128, D, 0, 1);    // V is MN-major
      // descriptors of the Q tiles and of ring slot 0; other slots / k-steps add offsets >> 4
      const uint64_t dq0 = umma_smem_desc(sQ, 16, 1024, kLayoutSW128);
      const uint64_t dk0 = umma_smem_desc(sRing, 16, 1024, kLayoutSW128);
      const uint64_t dv0 = umma_smem_desc(sRing, C::BLK, 1024, kLayoutSW128);
      auto issue_s = [&](int s, int sl) {
        const uint32_t d_t = tmem + C::col_s(s);
        const uint64_t a = dq0 + static_cast<uint64_t>((s * C::TILE) >> 4);
        const uint64_t bq = dk0 + static_cast<uint64_t>((sl * C::TILE) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t o = static_cast<uint64_t>(((k >> 2) * C::BLK + (k & 3) * 32) >> 4);
          umma_ss(d_t, a + o, bq + o, kIdescS, k > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int s, int sl, bool acc) {
        const uint32_t d_t = tmem + C::col_o(s);
        const uint32_t a_t = tmem + C::col_s(s);
        const uint64_t bv = dv0 + static_cast<uint64_t>((sl * C::TILE) >> 4);
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 128 keys, 16 per MMA
          umma_ts(d_t, a_t + 8 * k, bv + static_cast<uint64_t>((k * 2048) >> 4), kIdescO,
                  (acc || k > 0) ? 1u : 0u);
      };
      auto kslot = [](int j) { return (2 * j) % C::NSLOT; };
      auto kpar = [](int j) { return static_cast<uint32_t>(((2 * j) / C::NSLOT) & 1); };
      auto vslot = [](int j) { return (2 * j + 1) % C::NSLOT; };
      auto vpar = [](int j) { return static_cast<uint32_t>(((2 * j + 1) / C::NSLOT) & 1); };
      const long long lim = p.wait_limit;
      bool ok = mbar_wait(bar(C::B_FULL + kslot(0)), kpar(0), lim, abort_flag, p.status);
      ok = ok && mbar_wait(bar(C::B_QREADY + 0), 0, lim, abort_flag, p.status);
      if (ok) {
        issue_s(0, kslot(0));
        umma_commit(bar(C::B_SFULL + 0));
        if (ns == 2) {
          ok = mbar_wait(bar(C::B_QREADY + 1), 0, lim, abort_flag, p.status);
          if (ok) {
            issue_s(1, kslot(0));
            umma_commit(bar(C::B_SFULL + 1));
          }
        }
        umma_commit(bar(C::B_EMPTY + kslot(0)));
      }
      for (int j = 0; ok && j < n_it; ++j) {  // j counts visited tiles
        const bool has_next = j + 1 < n_it;
        RA_STAMP(0, j);
        if (!mbar_wait(bar(C::B_PFULL + 0), j & 1, lim, abort_flag, p.status) ||
            !mbar_wait(bar(C::B_FULL + vslot(j)), vpar(j), lim, abort_flag, p.status))
          break;
        tc_fence_after();
        RA_STAMP(1, j);
        issue_pv(0, vslot(j), j > 0);
        RA_STAMP(2, j);
        if (!has_next) umma_commit(bar(C::B_OFULL + 0));
        if (has_next) {
          if (!mbar_wait(bar(C::B_FULL + kslot(j + 1)), kpar(j + 1), lim, abort_flag, p.status))
            break;
          // (no tcgen05 fence: S reads only shared memory, synchronised by the mbarrier)
          RA_STAMP(3, j);
          issue_s(0, kslot(j + 1));
          RA_STAMP(4, j);
          umma_commit(bar(C::B_SFULL + 0));
        }
        if (ns == 2) {
          if (!mbar_wait(bar(C::B_PFULL + 1), j & 1, lim, abort_flag, p.status)) break;
          tc_fence_after();
          RA_STAMP(5, j);
          issue_pv(1, vslot(j), j > 0);
          RA_STAMP(6, j);
          if (!has_next) umma_commit(bar(C::B_OFULL + 1));
          umma_commit(bar(C::B_EMPTY + vslot(j)));
          if (has_next) {
            issue_s(1, kslot(j + 1));
            RA_STAMP(7, j);
            umma_commit(bar(C::B_SFULL + 1));
            umma_commit(bar(C::B_EMPTY + kslot(j + 1)));
          }
        } else {
          umma_commit(bar(C::B_EMPTY + vslot(j)));
          if (has_next) umma_commit(bar(C::B_EMPTY + kslot(j + 1)));
        }
      }
      // every MMA issued above must finish before TMEM is released
      umma_commit(bar(C::B_DRAIN));
      mbar_drain(bar(C::B_DRAIN), 0);
    }
    __syncwarp();
  }
  } else {
  regs_inc<208>();
  if ((warp >> 2) - 1 < ns) {
    // ================================================================ softmax warpgroups
    const int s = (warp >> 2) - 1;
    const int qd = warp & 3;
    const int r = qd * 32 + lane;  // query row within the tile == TMEM lane
    const int qrow = q0 + r;
    const uint32_t t_lane = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t tS = tmem + t_lane + C::col_s(s);
    const uint32_t tO = tmem + t_lane + C::col_o(s);
    const long long lim = p.wait_limit;

    // rotate the warp's 32 rows of Q_s in shared memory (128-byte swizzled layout of
    // the TMA box). D/8 lanes share a row, one 16-byte chunk (4 pairs) each, so every table
    // load of the warp reads whole consecutive table rows (coalesced); all loads of the warp
    // are issued before the first rotation.
    bool ok = mbar_wait_warp(bar(C::B_QFULL + s), 0, lim, abort_flag, p.status);
    if (ok) {
      constexpr int CPR = D / 8;        // 16-byte chunks per row
      constexpr int RPS = 32 / CPR;     // rows per warp step
      constexpr int NSTEP = 32 / RPS;   // steps for the warp's 32 rows
      const int k = lane % CPR, kb = k >> 3, c = k & 7;
      float4 t[NSTEP][2];
#pragma unroll
      for (int st = 0; st < NSTEP; ++st) {
        const int rr = qd * 32 + st * RPS + lane / CPR;
        const int qr = min(q0 + rr, p.Sq - 1);  // rows past Sq read a valid row, unused
        const float4* trow = reinterpret_cast<const float4*>(
            p.tab + static_cast<long long>(p.q_tab_off + qr) * (D / 2));
        t[st][0] = __ldg(trow + 2 * k);
        t[st][1] = __ldg(trow + 2 * k + 1);
      }
#pragma unroll
      for (int st = 0; st < NSTEP; ++st) {
        const int rr = qd * 32 + st * RPS + lane / CPR;
        if (q0 + rr < p.Sq) {
          uint4* ptr = reinterpret_cast<uint4*>(smem + C::OFF_Q + s * C::TILE + kb * C::BLK +
                                                rr * 128 + ((c ^ (rr & 7)) << 4));
          const float2 cs[4] = {make_float2(t[st][0].x, t[st][0].y),
                                make_float2(t[st][0].z, t[st][0].w),
                                make_float2(t[st][1].x, t[st][1].y),
                                make_float2(t[st][1].z, t[st][1].w)};
          *ptr = rotate8(*ptr, cs);
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(C::B_QREADY + s));

    float m = -INFINITY;  // running row max, in log2 units of the scaled score
    float l = 0.f;        // running row sum of 2^(x - m)
    const float sl2 = p.scale_log2;
    const int lim_causal = min(p.Sk - 1, qrow + off);
    for (int j = 0; ok && j < n_it; ++j) {  // j counts visited tiles; KV tile j_lo + j
      if (!mbar_wait_warp(bar(C::B_SFULL + s), j & 1, lim, abort_flag, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0 && qd == 0) RA_STAMP(8 + 2 * s, j);
      uint32_t sr[128];
      tmem_ld32(tS + 0, sr + 0);
      tmem_ld32(tS + 32, sr + 32);
      tmem_ld32(tS + 64, sr + 64);
      tmem_ld32(tS + 96, sr + 96);
      tmem_wait_ld();

      // causal / sequence-end mask, only on tiles that reach past some row's limit
      const int kbase = (j_lo + j) * 128;
      const bool need_mask = (kbase + 128 > p.Sk) || (p.causal && kbase + 127 > q0 + off) ||
                             (p.window > 0 && kbase + p.window < q0 + 128 + off);
      if (need_mask) {
        const int lim_k = (p.causal ? lim_causal : p.Sk - 1) - kbase;
        const int lo_k = (p.window > 0) ? qrow + off - p.window + 1 - kbase : 0;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim_k || c < lo_k) sr[c] = 0xff800000u;  // -inf
      }
      // online softmax with a lazily updated reference max m. Once a row has a
      // reference, P is computed speculatively with it while the tile max is gathered
      // on the side; only if some row's max grew by more than 8 (log2 units) does the warp
      // redo the tile exactly (rescale O, P with the new reference). Either way every row
      // ends with the same values as the plain max-first order.
      float rs = 0.f;
      bool done = false;
      float mt = -INFINITY;
      if (!__any_sync(0xffffffffu, m == -INFINITY)) {
        rs = need_mask ? softmax_p_store_max<0>(sr, sl2, m, tS, mt)
                       : softmax_p_store_max<kEmuPairs>(sr, sl2, m, tS, mt);
        done = !__any_sync(0xffffffffu, fmaxf(m, mt * sl2) > m + 8.0f);
      } else {
        // tile max of the raw scores: eight independent 3-input max chains, then a tree
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mx[k] = max3f(__uint_as_float(sr[k]), __uint_as_float(sr[k + 8]),
                        __uint_as_float(sr[k + 16]));
#pragma unroll
        for (int c = 24; c < 120; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mx[k] = max3f(mx[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], __uint_as_float(sr[120 + k]));
        mt = max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      }
      if (!done) {
        const float m_new = fmaxf(m, mt * sl2);
        // Keep the old reference unless the max grew by more than 8 (P stays <= 256);
        // O / l is exact for any common reference, so skipping the rescale is lossless.
        const bool upd = m_new > m + 8.0f;
        const float alpha = upd ? ex2(m - m_new) : 1.0f;
        if (upd) m = m_new;
        l *= alpha;
        if (j > 0 && __any_sync(0xffffffffu, upd)) {
          // O_s *= alpha (PV_s(j-1) has completed: it was issued before S_s(j))
#pragma unroll
          for (int cb = 0; cb < D; cb += 32) {
            uint32_t o[32];
            tmem_ld32(tO + cb, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + cb, o);
          }
        }
        // p = 2^(s * log2(e)/sqrt(D) - m) -> bf16 P over the S columns; a row that has seen
        // no allowed key yet (only under a window) keeps m = -inf and gets P = 0
        const float m_use = (m == -INFINITY) ? 0.f : m;
        rs = need_mask ? softmax_p_store<0>(sr, sl2, m_use, tS)
                       : softmax_p_store<kEmuPairs>(sr, sl2, m_use, tS);
      }
      l += rs;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_PFULL + s));
      if (lane == 0 && qd == 0) RA_STAMP(9 + 2 * s, j);
    }

    // epilogue, partial mode: O / l and the LSE in fp32, merged with the running result
    // (weights exp(lse - merged lse) on each side); every row has at least one allowed key
    if (p.o_acc != nullptr) {
      if (ok && mbar_wait_warp(bar(C::B_OFULL + s), 0, lim, abort_flag, p.status)) {
        tc_fence_after();
        const long long row = static_cast<long long>(b * p.Hq + h0 + s) * p.acc_rows + qrow;
        const float lse_new = (m + log2f(l)) * kLn2;
        float w_old = 0.f, w_new = 1.0f / l, lse_out = lse_new;
        if (p.accumulate && qrow < p.Sq) {
          const float lse_old = p.lse_acc[row];
          if (lse_old != -INFINITY) {
            const float mx = fmaxf(lse_old, lse_new);
            const float eo = expf(lse_old - mx), en = expf(lse_new - mx);
            const float den = eo + en;
            w_old = eo / den;
            w_new = en / (den * l);
            lse_out = mx + logf(den);
          }
        }
        float4* acc = reinterpret_cast<float4*>(p.o_acc + row * D);
        __nv_bfloat16* orow = p.out ? p.out + row * D : nullptr;
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t o[32];
          tmem_ld32(tO + cb, o);
          tmem_wait_ld();
          if (qrow < p.Sq) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * w_new;
            if (w_old != 0.f) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 a = acc[cb / 4 + i];
                v[4 * i + 0] += w_old * a.x;
                v[4 * i + 1] += w_old * a.y;
                v[4 * i + 2] += w_old * a.z;
                v[4 * i + 3] += w_old * a.w;
              }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
              acc[cb / 4 + i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            if (orow) {
              uint4* dst = reinterpret_cast<uint4*>(orow + cb);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pack_bf16(v[8 * i + 0], v[8 * i + 1]),
                                    pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                                    pack_bf16(v[8 * i + 4], v[8 * i + 5]),
                                    pack_bf16(v[8 * i + 6], v[8 * i + 7]));
            }
          }
        }
        if (qrow < p.Sq) p.lse_acc[row] = lse_out;
      }
    } else if (ok && mbar_wait_warp(bar(C::B_OFULL + s), 0, lim, abort_flag, p.status)) {
      // epilogue O / l -> bf16
      tc_fence_after();
      const float inv = 1.0f / l;
      const uint64_t pol_out = l2_policy_evict_first();
      __nv_bfloat16* orow =
          p.out + (static_cast<long long>(b * p.Hq + h0 + s) * p.Sq + qrow) * D;
#pragma unroll
      for (int cb = 0; cb < D; cb += 32) {
        uint32_t o[32];
        tmem_ld32(tO + cb, o);
        tmem_wait_ld();
        if (qrow < p.Sq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cb);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
            st_global_v4_hint(dst + i, w, pol_out);
          }
        }
      }
    }
  }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace ra
