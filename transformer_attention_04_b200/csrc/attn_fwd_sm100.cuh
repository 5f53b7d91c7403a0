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
// Persistent kernel: one CTA per SM walks a list of work units. A unit is two 128-row query
// tiles ("slots") that share every K/V tile: two query heads of the same KV group at the
// same positions (GQA with an even group size), or, for odd group sizes (MHA included), two
// consecutive query tiles of one head (the first tile's rows see one more key tile than
// they may, which the causal mask zeroes).
// Units are ordered longest causal extent first and dealt to the CTAs in snake order
// (round k runs forward over the CTAs when k is even, backward when odd), which balances the
// causal triangle. Warp roles (384 threads):
//   warp 0        TMA producer: the Q tiles of each unit into one of two Q buffers, and the
//                 K'/V tiles of every unit, in order, through an NSLOT-deep ring.
//   warp 1        TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 2-3     RoPE rotation of each unit's Q tiles in shared memory, done while the
//                 previous unit runs.
//   warps 4-7     softmax warpgroup of slot 0 (thread = query row = TMEM lane); after a
//                 unit's last tile it writes the unit's output from TMEM into the slot's
//                 finished Q tile in shared memory, and one of its threads stores the tile
//                 with TMA (an fp32 merge into the running result in partial mode).
//   warps 8-11    softmax warpgroup of slot 1.
// Per KV tile j the issuer runs S_s = Q_s K_j^T (SS MMA, fp32 in TMEM), the softmax group
// turns S_s into bf16 P_s written over the same TMEM columns, and the issuer runs
// O_s += P_s V_j with P taken from TMEM (TS MMA). The issue order PV0 S0' PV1 S1' ... runs
// on across unit boundaries (S' being the first S of the next unit after a unit's last
// tile), so one slot's softmax always overlaps the other slot's MMAs. tcgen05.mma issued by
// one thread execute in order, so S_s(j+1) never overwrites P_s(j) before PV_s(j) has read
// it, and each commit after S_s(j) also covers PV_s(j-1) (used before rescaling O_s).
//
// K is rotated once per call by rope_rotate_kernel into a workspace, since every K tile is
// re-read by S/128 query tiles; each Q tile is read by one unit and is rotated in shared
// memory after its TMA load.
#pragma once

#include "ptx.cuh"
#include "rope.cuh"

namespace ra {

constexpr float kLn2 = 0.6931471805599453f;
constexpr int kFwdThreads = 384;  // the kernel's block size (12 warps, roles below)

struct FwdParams {
  __nv_bfloat16* out;   // [B, Hq, Sq, D]
  const float2* tab;    // RoPE (cos, sin) table, D/2 entries per query row position
  unsigned int* status; // sticky device status word
  long long wait_limit; // polls per mbarrier wait before giving up
  int B, Hq, Hkv, Sq, Sk;
  int G;                // Hq / Hkv
  int n_slots;          // query tiles per unit (1 or 2)
  int pair_q;           // 1: the slots are two consecutive query tiles of one head (odd G);
                        // 0: the same query tile of two heads of the KV group (even G)
  int ppg;              // units per (batch, KV group, query-tile group)
  int n_qtiles;         // ceil(Sq / 128)
  int n_units;          // n_qtiles * B * Hkv * ppg
  int causal;
  int off;              // query row i sits at key index i + off (causal: key j allowed iff j <= i + off)
  int off2;             // the same for the rows of the second query segment (i >= q_split)
  int window;           // 0 = none; else key j is allowed to query row i iff j > i + off - window
  int q_tab_off;        // query row i < q_split reads table row q_tab_off + i
  int q_split;          // first row of a second segment of positions (Sq if none)...
  int q_tab_off2;       // ...whose row i reads table row q_tab_off2 + i
  float scale_log2;     // log2(e) / sqrt(D)
  float rope_base;
  // partial (ring) mode when o_acc is set: O / l in fp32 [B, Hq, Sq, D] and the row's natural
  // log-sum-exp in lse_acc [B, Hq, Sq], merged into their contents when accumulate is set;
  // `out` (bf16) is then optional and receives the merged result
  float* o_acc;
  float* lse_acc;
  int accumulate;
  int acc_rows;  // partial mode: rows between heads in o_acc / lse_acc / out (>= Sq)
  int dep_late;  // partial mode: the inputs were complete before the previous kernel started;
                 // wait for that kernel only before merging into the running result
};

template <int D>
struct FwdCfg {
  static constexpr int KB = D / 64;                  // 128-byte column blocks per row
  static constexpr int BLK = 128 * 128;              // bytes of one 128-row column block
  static constexpr int TILE = 128 * D * 2;           // bytes of one 128 x D bf16 tile
  // Two Q buffers of two tiles each (the next unit's Q loads and is rotated while the
  // current unit runs). K and V tiles stream through one ring in the order K0 V0 K1 V1 ...:
  // 3 slots at D = 128 (4 Q tiles + 3 slots = 224 KB of shared memory). A K tile's slot is
  // refilled one tile period before its S needs it, which covers the TMA latency.
  static constexpr int NSLOT = (D == 128) ? 3 : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + 4 * TILE;
  static constexpr int OFF_BAR = OFF_RING + NSLOT * TILE;
  static constexpr int SMEM = OFF_BAR + 512;  // the dynamic shared base is 1024-aligned (checked)
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns: S/P of slot s at 128*s, O of slot s at 256 + D*s
  __device__ static constexpr uint32_t col_s(int s) { return 128u * static_cast<uint32_t>(s); }
  __device__ static constexpr uint32_t col_o(int s) { return 256u + static_cast<uint32_t>(D * s); }
  // barrier indices (8 bytes each); [b] = Q buffer, [s] = slot
  static constexpr int B_QFULL = 0,    // [b]: both Q tiles of a unit landed (TMA)
      B_QREADY = 2,                    // [b]: rotated (2 rotating warps)
      B_QEMPTY = 4,                    // [b]: the unit's last S read it (MMA commit)
      B_SFULL = 6,                     // [s]: S_s in TMEM
      B_PFULL = 8,                     // [s]: P_s in TMEM (4 softmax warps)
      B_OFULL = 10,                    // [s]: the unit's last PV_s done
      B_DRAIN = 12,
      B_QSTAGED = 13,                  // [b]: the unit's outputs, staged in its Q tiles, stored
      B_EPI = 15,                      // [s]: slot s's rows staged (4 softmax warps)
      B_FULL = 17, B_EMPTY = 17 + NSLOT, N_BAR = 17 + 2 * NSLOT;
  static constexpr int OFF_TMEM_SLOT = 8 * N_BAR;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
  static_assert(OFF_ABORT + 4 <= 512, "barrier area");
  static_assert(SMEM <= 232448, "shared memory per block");
};

// One work unit: which query tile(s), heads and KV tiles. Slot s holds query rows
// q0 + dq(s) .. + 127 of head h0 + dh(s).
struct Unit {
  int b, h0, kv_bh, q0, j_lo, n_it;
};
__device__ __forceinline__ int slot_dq(const FwdParams& p, int s) { return p.pair_q ? 128 * s : 0; }
__device__ __forceinline__ int slot_dh(const FwdParams& p, int s) { return p.pair_q ? 0 : s; }

// Unit u of the longest-first order: rank t of the query-tile groups (one tile, or two
// consecutive tiles with pair_q; causal: the last group first), then batch, KV group and
// head (pair).
__device__ __forceinline__ Unit unit_at(const FwdParams& p, int u) {
  Unit w;
  const int per_tile = p.B * p.Hkv * p.ppg;
  const int t_rank = u / per_tile;
  const int rem = u - t_rank * per_tile;
  const int n_groups = p.pair_q ? (p.n_qtiles + 1) / 2 : p.n_qtiles;
  const int qg = p.causal ? (n_groups - 1 - t_rank) : t_rank;
  w.b = rem / (p.Hkv * p.ppg);
  const int g = (rem / p.ppg) % p.Hkv;
  w.h0 = g * p.G + (rem % p.ppg) * (p.pair_q ? 1 : p.n_slots);
  w.kv_bh = w.b * p.Hkv + g;
  w.q0 = qg * 128 * (p.pair_q ? 2 : 1);
  const int q_last = w.q0 + slot_dq(p, p.n_slots - 1) + 127;  // the unit's last query row
  int n_kv = (p.Sk + 127) / 128;
  // a unit lies in one query segment (the host keeps q_split a multiple of its rows)
  const int off = (w.q0 >= p.q_split) ? p.off2 : p.off;
  if (p.causal) n_kv = min(n_kv, (min(p.Sq - 1, q_last) + off) / 128 + 1);
  // with a sliding window, tiles wholly below the first row's window are skipped too
  w.j_lo = (p.window > 0) ? max(0, w.q0 + off - p.window + 1) / 128 : 0;
  w.n_it = n_kv - w.j_lo;  // KV tiles visited: j_lo .. n_kv - 1
  return w;
}

// The k-th unit of this CTA in snake order, or -1 past the end.
__device__ __forceinline__ int unit_of(const FwdParams& p, int k) {
  const int P = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int u = k * P + ((k & 1) ? (P - 1 - c) : c);
  return u < p.n_units ? u : -1;
}

// P = 2^(s * sl2 - m) for one 128-column row of S held in registers; writes the bf16 P
// over the first 64 TMEM columns at tS and returns the row sum of the fp32 values.
// Pairs go through one packed FMA; the exponentials run on the MUFU.
__device__ __forceinline__ float softmax_p_store(const uint32_t* sr, float sl2, float m,
                                                 uint32_t tS) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m, -m);
  uint64_t acc2[2] = {0, 0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t pk[32];
#pragma unroll
    for (int c2 = 0; c2 < 32; ++c2) {
      const int c = h * 64 + 2 * c2;
      const uint64_t x2 =
          f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm2);
      float x0, x1;
      f2_unpack(x2, x0, x1);
      const float p0 = ex2(x0), p1 = ex2(x1);
      acc2[c2 & 1] = f2_add(acc2[c2 & 1], f2_pack(p0, p1));
      pk[c2] = pack_bf16(p0, p1);
    }
    tmem_st32(tS + 32 * h, pk);
  }
  const uint64_t a = f2_add(acc2[0], acc2[1]);
  float a0, a1;
  f2_unpack(a, a0, a1);
  return a0 + a1;
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
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
  const int ns = p.n_slots;
  const long long lim = p.wait_limit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_QFULL + i), 1);
      mbar_init(bar(C::B_QREADY + i), 2);  // one arrival per rotating warp
      mbar_init(bar(C::B_QEMPTY + i), 1);
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 4);   // one arrival per softmax warp
      mbar_init(bar(C::B_OFULL + i), 1);
      // one TMA store per slot, or (partial mode) one arrival per softmax warp
      mbar_init(bar(C::B_QSTAGED + i), p.o_acc != nullptr ? 4 * ns : ns);
      mbar_init(bar(C::B_EPI + i), 4);
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
  // Only a chained ring block (dep_late) is launched with a programmatic dependency on the
  // kernel before it (the previous block): it reads only inputs that were complete before that
  // kernel started and waits before its first merge. Other launches are plain, where this wait
  // returns at once. Either way the next launch, a chained block, may start its set-up.
  if (!p.dep_late) grid_dep_wait();
  grid_dep_launch();

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
      int i = 0;             // ring items issued: tile i/2 of K (i even) or V (i odd), slot i % NSLOT
      int q_issued0 = 0, q_issued1 = 0;  // Q loads issued into buffers 0 and 1
      bool ok = true;
      auto load_q = [&](int k) -> bool {  // Q tiles of this CTA's k-th unit into buffer k & 1
        const int u = unit_of(p, k);
        if (u < 0) return true;
        const int qb = k & 1;
        // the buffer's previous unit (k - 2) must have issued its last S
        if (k >= 2 && !mbar_wait(bar(C::B_QEMPTY + qb), ((k - 2) >> 1) & 1, lim, abort_flag,
                                 p.status))
          return false;
        // unit k - 2's outputs were staged in this buffer: it has been read out
        if (k >= 2 &&
            !mbar_wait(bar(C::B_QSTAGED + qb), ((k - 2) >> 1) & 1, lim, abort_flag, p.status))
          return false;
        const Unit w = unit_at(p, u);
        mbar_expect_tx(bar(C::B_QFULL + qb), ns * C::TILE);
        for (int s = 0; s < ns; ++s)
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_3d_hint(sQ + (qb * 2 + s) * C::TILE + kb * C::BLK, &tm_q, kb * 64,
                             w.q0 + slot_dq(p, s), w.b * p.Hq + w.h0 + slot_dh(p, s),
                             bar(C::B_QFULL + qb), pol_once);
        if (qb) ++q_issued1; else ++q_issued0;
        return true;
      };
      auto load_kv = [&](const Unit& w, int jj, int kv) -> bool {  // kv 0: K, 1: V
        const int sl = i % C::NSLOT;
        const int j = i - C::NSLOT;  // the slot's previous item
        if constexpr (C::NSLOT % 2 == 1) {
          // K and V items alternate in each slot. A V tile is released by its own commit after
          // its last PV (EMPTY completes once per V occupant); a K tile by the last S that reads
          // it (the SFULL commit of the tile's last slot). K(t)'s release is checked right after
          // K(t + 1) has been issued, and SFULL's next phase needs K(t + 1) to land: the barrier
          // is at most one phase past the one awaited.
          if (j >= 0 && !((j & 1) ? mbar_wait(bar(C::B_EMPTY + sl), ((j / C::NSLOT) >> 1) & 1,
                                              lim, abort_flag, p.status)
                                  : mbar_wait(bar(C::B_SFULL + ns - 1), (j >> 1) & 1, lim,
                                              abort_flag, p.status)))
            return false;
        } else {
          // an even ring keeps K and V in separate slots, several tiles ahead: every item is
          // released by a commit of its own
          if (j >= 0 && !mbar_wait(bar(C::B_EMPTY + sl), (j / C::NSLOT) & 1, lim, abort_flag,
                                   p.status))
            return false;
        }
        mbar_expect_tx(bar(C::B_FULL + sl), C::TILE);
        const CUtensorMap* map = kv ? &tm_v : &tm_k;
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d_hint(sRing + sl * C::TILE + kb * C::BLK, map, kb * 64, (w.j_lo + jj) * 128,
                           w.kv_bh, bar(C::B_FULL + sl), pol_keep);
        ++i;
        return true;
      };
      // (partial mode, merging) the accumulator rows the unit's epilogue reads, brought into
      // L2 a few tiles ahead so that its loads do not wait on DRAM
      auto prefetch_acc = [&](const Unit& w) {
        for (int s = 0; s < ns; ++s) {
          const int q0s = w.q0 + slot_dq(p, s);
          const int nrows = min(128, p.Sq - q0s);
          if (nrows <= 0) continue;
          const long long row0 =
              static_cast<long long>(w.b * p.Hq + w.h0 + slot_dh(p, s)) * p.acc_rows + q0s;
          bulk_prefetch_l2(p.o_acc + row0 * D, static_cast<uint32_t>(nrows * D * 4));
          // the rows' LSE: every 128-byte line of [row0, row0 + nrows)
          for (int j = 0; j < nrows; j += 32) prefetch_l2_line(p.lse_acc + row0 + j);
          prefetch_l2_line(p.lse_acc + row0 + nrows - 1);
        }
      };
      const bool merging = p.o_acc != nullptr && p.accumulate;
      ok = load_q(0);
      for (int k = 0; ok && unit_of(p, k) >= 0; ++k) {
        const Unit w = unit_at(p, unit_of(p, k));
        const int jp = max(0, w.n_it - 3);  // the tile whose loads carry the prefetch
        // this unit's first K/V tile, then the next unit's Q (its buffer frees once the
        // unit before this one has issued its last S), then the rest of this unit's tiles
        ok = load_kv(w, 0, 0) && load_kv(w, 0, 1) && load_q(k + 1);
        if (ok && merging && jp == 0) prefetch_acc(w);
        for (int jj = 1; ok && jj < w.n_it; ++jj) {
          ok = load_kv(w, jj, 0) && load_kv(w, jj, 1);
          if (ok && merging && jj == jp) prefetch_acc(w);
        }
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA can exit
        if (q_issued0) mbar_drain(bar(C::B_QFULL + 0), (q_issued0 - 1) & 1);
        if (q_issued1) mbar_drain(bar(C::B_QFULL + 1), (q_issued1 - 1) & 1);
        for (int j = max(0, i - C::NSLOT); j < i; ++j)
          mbar_drain(bar(C::B_FULL + j % C::NSLOT), (j / C::NSLOT) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // One thread issues every MMA, in the order PV0(t) S0(t+1) PV1(t) S1(t+1) per tile t
    // (S(t+1) being the S of the unit's next tile, or the next unit's first). The single
    // order makes the two slots alternate: one slot's softmax runs while the other slot's
    // MMAs execute. Each tcgen05.mma holds the issuing thread for about its duration and
    // each barrier wait or commit costs it a few hundred cycles even when the phase has long
    // completed, so the thread keeps the code between MMAs short and polls the tile's V, the
    // next K and P0 together: one round trip instead of three (the tensor pipe idles through
    // every one of them).
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_bf16(128, 128, 0, 0);  // Q, K both K-major
      constexpr uint32_t kIdescO = umma_idesc_bf16(128, D, 0, 1);    // V is MN-major
      constexpr uint32_t kHi = umma_desc_hi_sw128(1024);
      // low descriptor words of Q tile 0 and of ring slot 0 (as the B operand of S, and as V
      // for PV); other tiles and slots add a multiple of TILE >> 4
      const uint32_t q_lo0 = umma_desc_lo(sQ, 16);
      const uint32_t k_lo0 = umma_desc_lo(sRing, 16);
      const uint32_t v_lo0 = umma_desc_lo(sRing, C::BLK);
      auto issue_s = [&](int qtile, int s, int sl) {  // qtile = Q buffer * 2 + slot
        const uint32_t d_t = tmem + C::col_s(s);
        const uint32_t qlo = q_lo0 + static_cast<uint32_t>(qtile * (C::TILE >> 4));
        const uint32_t klo = k_lo0 + static_cast<uint32_t>(sl * (C::TILE >> 4));
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          constexpr uint32_t kBlk = C::BLK >> 4;
          const uint32_t o = static_cast<uint32_t>((k >> 2) * kBlk + (k & 3) * 2);
          umma_ss(d_t, umma_desc(qlo + o, kHi), umma_desc(klo + o, kHi), kIdescS, k > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int s, int sl, bool acc) {
        const uint32_t d_t = tmem + C::col_o(s);
        const uint32_t a_t = tmem + C::col_s(s);
        const uint32_t vlo = v_lo0 + static_cast<uint32_t>(sl * (C::TILE >> 4));
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 128 keys, 16 per MMA
          umma_ts(d_t, a_t + 8 * k, umma_desc(vlo + static_cast<uint32_t>(k * (2048 >> 4)), kHi),
                  kIdescO, (acc || k > 0) ? 1u : 0u);
      };
      // global tile t: K item 2t, V item 2t + 1
      auto slot = [](int item) { return item % C::NSLOT; };
      auto par = [](int item) { return static_cast<uint32_t>((item / C::NSLOT) & 1); };
      auto wait = [&](int b, uint32_t parity) {
        return mbar_wait(bar(b), parity, lim, abort_flag, p.status);
      };

      bool ok = false;
      int n_it = 0;
      const int u0 = unit_of(p, 0);
      if (u0 >= 0) {
        n_it = unit_at(p, u0).n_it;
        // S of unit 0's first tile
        ok = wait(C::B_QREADY + 0, 0) && wait(C::B_FULL + slot(0), par(0));
        if (ok) {
          issue_s(0, 0, slot(0));
          umma_commit(bar(C::B_SFULL + 0));
          if (ns == 2) {
            issue_s(1, 1, slot(0));
            umma_commit(bar(C::B_SFULL + 1));
          }
          if (n_it == 1) umma_commit(bar(C::B_QEMPTY + 0));
          if constexpr (C::NSLOT % 2 == 0) umma_commit(bar(C::B_EMPTY + slot(0)));
        }
      }
      int t = 0;
      for (int k = 0; ok; ++k) {
        const int nu = unit_of(p, k + 1);
        const int n_next = nu >= 0 ? unit_at(p, nu).n_it : 0;
        for (int jj = 0; ok && jj < n_it; ++jj, ++t) {
          const bool last = jj + 1 == n_it;
          const bool has_next = !last || n_next > 0;
          const int qbn = last ? (k + 1) & 1 : k & 1;                  // Q buffer of the next tile
          const bool next_last = last ? n_next == 1 : jj + 2 == n_it;  // next tile ends its unit
          // the tile's V, the next K and P0 polled together (the next unit's Q first)
          ok = (!(has_next && last) || wait(C::B_QREADY + qbn, ((k + 1) >> 1) & 1)) &&
               mbar_wait3(bar(C::B_PFULL + 0), t & 1, bar(C::B_FULL + slot(2 * t + 1)),
                          par(2 * t + 1), bar(C::B_FULL + slot(2 * t + 2)), par(2 * t + 2),
                          has_next ? 3 : 2, lim, abort_flag, p.status);
          if (!ok) break;
          // ---- slot 0: PV0(t), then S0(t + 1)
          // (P_s of a unit's first tile comes after the softmax group has read the previous
          // unit's O_s, so PV_s may overwrite it)
          tc_fence_after();
          issue_pv(0, slot(2 * t + 1), jj > 0);
          if (last) umma_commit(bar(C::B_OFULL + 0));
          if (has_next) {
            issue_s(qbn * 2 + 0, 0, slot(2 * t + 2));
            umma_commit(bar(C::B_SFULL + 0));
          }
          // ---- slot 1: PV1(t), then S1(t + 1)
          if (ns == 2) {
            if (!wait(C::B_PFULL + 1, t & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(1, slot(2 * t + 1), jj > 0);
            if (last) umma_commit(bar(C::B_OFULL + 1));
            umma_commit(bar(C::B_EMPTY + slot(2 * t + 1)));
            if (has_next) {
              issue_s(qbn * 2 + 1, 1, slot(2 * t + 2));
              umma_commit(bar(C::B_SFULL + 1));
            }
          }
          if (ns == 1) umma_commit(bar(C::B_EMPTY + slot(2 * t + 1)));
          if (has_next) {
            if (next_last) umma_commit(bar(C::B_QEMPTY + qbn));  // that unit's last S
            if constexpr (C::NSLOT % 2 == 0) umma_commit(bar(C::B_EMPTY + slot(2 * t + 2)));
          }
        }
        if (!ok || n_next == 0) break;
        n_it = n_next;
      }
      // every MMA issued above must finish before TMEM is released
      umma_commit(bar(C::B_DRAIN));
      mbar_drain(bar(C::B_DRAIN), 0);
    }
    __syncwarp();
  } else {
    // ================================================================ Q rotation (warps 2-3)
    // Each unit's Q tiles are rotated in shared memory once they land, while the previous
    // unit runs; the MMA issuer waits for them only at the unit's first S.
    // Rotation split: thread rt owns 16-byte chunk ck (4 pairs) of a block of RB consecutive
    // rows; it takes the (cos, sin) of the block's first row from the table and steps to
    // the next row with the angle-addition formula, since consecutive rows differ by one
    // position.
    const int rt = (warp - 2) * 32 + lane;  // 0..63
    constexpr int CPR = D / 8;              // chunks per row
    constexpr int RB = 128 * CPR / 64;      // rows per block: 64 threads cover 128 rows
    const int ck = rt % CPR, rb0 = (rt / CPR) * RB;
    float2 step[4];  // (cos, sin) of theta_i for the chunk's four pairs, exact in fp64 first
    {
      const double log2_base = log2(static_cast<double>(p.rope_base));
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = ck * 4 + e;
        const double theta = exp2(-(2.0 * i / D) * log2_base);
        double sd, cd;
        sincos(theta, &sd, &cd);
        step[e] = make_float2(static_cast<float>(cd), static_cast<float>(sd));
      }
    }
    auto rotate_unit = [&](int k) -> bool {
      const int u = unit_of(p, k);
      if (u < 0) return true;
      const int qb = k & 1;
      if (!mbar_wait_warp(bar(C::B_QFULL + qb), (k >> 1) & 1, lim, abort_flag, p.status))
        return false;
      const Unit w = unit_at(p, u);
      const int kb = ck >> 3, c = ck & 7;
      // slots at the same positions (two heads) share one pass; paired query tiles take one
      // pass each
      const int per_pass = p.pair_q ? 1 : ns;
      for (int s0 = 0; s0 < ns; s0 += per_pass) {
      float2 cs[4];
#pragma unroll 1
      for (int rr = 0; rr < RB; ++rr) {
        const int row = rb0 + rr, qr = w.q0 + slot_dq(p, s0) + row;
        if (qr >= p.Sq) break;
        if (rr == 0 || qr == p.q_split) {
          const int trow = (qr < p.q_split ? p.q_tab_off : p.q_tab_off2) + qr;
          const float4* t4 = reinterpret_cast<const float4*>(
              p.tab + static_cast<long long>(trow) * (D / 2) + ck * 4);
          const float4 a = __ldg(t4), b2 = __ldg(t4 + 1);
          cs[0] = make_float2(a.x, a.y);
          cs[1] = make_float2(a.z, a.w);
          cs[2] = make_float2(b2.x, b2.y);
          cs[3] = make_float2(b2.z, b2.w);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            cs[e] = make_float2(cs[e].x * step[e].x - cs[e].y * step[e].y,
                                cs[e].y * step[e].x + cs[e].x * step[e].y);
        }
        const uint32_t off = kb * C::BLK + row * 128 + ((c ^ (row & 7)) << 4);
        for (int s = s0; s < s0 + per_pass; ++s) {
          uint4* ptr = reinterpret_cast<uint4*>(smem + C::OFF_Q + (qb * 2 + s) * C::TILE + off);
          *ptr = rotate8(*ptr, cs);
        }
      }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::B_QREADY + qb));
      return true;
    };
    bool ok = true;
    for (int k = 0; ok && unit_of(p, k) >= 0; ++k) ok = rotate_unit(k);
  }
  } else {
  regs_inc<208>();
  if ((warp >> 2) - 1 < ns) {
    // ================================================================ softmax warpgroups
    const int s = (warp >> 2) - 1;
    const int qd = warp & 3;
    const int r = qd * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t t_lane = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t tS = tmem + t_lane + C::col_s(s);
    const uint32_t tO = tmem + t_lane + C::col_o(s);
    const float sl2 = p.scale_log2;
    bool ok = true;
    int t = 0;  // global tile counter
    for (int k = 0; ok && unit_of(p, k) >= 0; ++k) {
      const Unit w = unit_at(p, unit_of(p, k));
      const int q0s = w.q0 + slot_dq(p, s);  // this slot's first query row
      const int qrow = q0s + r;
      const int head = w.h0 + slot_dh(p, s);
      float m = -INFINITY;  // running row max, in log2 units of the scaled score
      float l = 0.f;        // running row sum of 2^(x - m)
      const int off = (q0s >= p.q_split) ? p.off2 : p.off;  // this slot's query segment
      const int lim_causal = min(p.Sk - 1, qrow + off);
      for (int jj = 0; jj < w.n_it; ++jj, ++t) {  // KV tile j_lo + jj
        if (!mbar_wait_warp(bar(C::B_SFULL + s), t & 1, lim, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(tS + 0, sr + 0);
        tmem_ld32(tS + 32, sr + 32);
        tmem_ld32(tS + 64, sr + 64);
        tmem_ld32(tS + 96, sr + 96);
        tmem_wait_ld();

        // causal / window / sequence-end mask, only on tiles that reach past some row's limit
        const int kbase = (w.j_lo + jj) * 128;
        const bool need_mask = (kbase + 128 > p.Sk) ||
                               (p.causal && kbase + 127 > q0s + off) ||
                               (p.window > 0 && kbase + p.window < q0s + 128 + off);
        if (need_mask) {
          const int lim_k = (p.causal ? lim_causal : p.Sk - 1) - kbase;
          const int lo_k = (p.window > 0) ? qrow + off - p.window + 1 - kbase : 0;
          // the sign of (lim_k - c) | (c - lo_k) masks the element: integer ops, no branch or
          // predicate (the limits differ from lane to lane)
          if (p.window > 0) {
#pragma unroll
            for (int c = 0; c < 128; ++c) {
              const uint32_t mk = static_cast<uint32_t>(((lim_k - c) | (c - lo_k)) >> 31);
              sr[c] = (sr[c] & ~mk) | (0xff800000u & mk);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 128; ++c) {
              const uint32_t mk = static_cast<uint32_t>((lim_k - c) >> 31);
              sr[c] = (sr[c] & ~mk) | (0xff800000u & mk);
            }
          }
        }
        // online softmax with a lazily updated reference max m. Once a row has a
        // reference, P is computed speculatively with it; every p is then at most 2^8 unless
        // the tile's row sum exceeds 2^8. Only then does the warp take the tile's max and, if
        // some row's max grew by more than 8 (log2 units), redo the tile exactly (rescale O,
        // P with the new reference). Either way every row ends with the same values as the
        // plain max-first order.
        float rs = 0.f;
        bool done = false, spec = false;
        float mt = -INFINITY;
        if (!__any_sync(0xffffffffu, m == -INFINITY)) {
          rs = softmax_p_store(sr, sl2, m, tS);
          spec = true;
          // every p <= 2^8 unless the tile's row sum exceeds 2^8 (or is inf / NaN)
          done = !__any_sync(0xffffffffu, !(rs <= 256.0f));
        }
        if (!done) {
          // tile max of the raw scores: eight independent 3-input max chains, then a tree
          float mx[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            mx[c] = max3f(__uint_as_float(sr[c]), __uint_as_float(sr[c + 8]),
                          __uint_as_float(sr[c + 16]));
#pragma unroll
          for (int c = 24; c < 120; c += 16)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              mx[e] = max3f(mx[e], __uint_as_float(sr[c + e]), __uint_as_float(sr[c + 8 + e]));
#pragma unroll
          for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], __uint_as_float(sr[120 + e]));
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
          if (jj > 0 && __any_sync(0xffffffffu, upd)) {
            // O_s *= alpha (PV_s(jj-1) has completed: it was issued before S_s(jj))
#pragma unroll
            for (int cb = 0; cb < D; cb += 32) {
              uint32_t o[32];
              tmem_ld32(tO + cb, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + cb, o);
            }
          }
          // p = 2^(s * log2(e)/sqrt(D) - m) -> bf16 P over the S columns; a row that has seen
          // no allowed key yet (only under a window) keeps m = -inf and gets P = 0. A
          // speculative P whose reference no row of the warp moved is already that P: a row
          // whose reference came from a few keys (a window's first tile) often sums past 2^8
          // without its max growing by 8.
          if (!spec || __any_sync(0xffffffffu, upd)) {
            const float m_use = (m == -INFINITY) ? 0.f : m;
            rs = softmax_p_store(sr, sl2, m_use, tS);
          }
        }
        l += rs;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_PFULL + s));
      }
      if (!ok) break;
      // ---- epilogue of the unit: once its last PV_s has completed, O_s is read out of TMEM
      // before this warpgroup's next P (and so before the next unit's first PV_s) exists
      auto wait_o = [&]() -> bool {
        if (!mbar_wait_warp(bar(C::B_OFULL + s), k & 1, lim, abort_flag, p.status)) return false;
        tc_fence_after();
        return true;
      };
      if (p.o_acc != nullptr) {
        if (p.dep_late) grid_dep_wait();  // the previous kernel's merges are complete
        // partial mode: O / l and the LSE in fp32, merged with the running result
        // (weights exp(lse - merged lse) on each side); every row has at least one allowed key
        const long long row = static_cast<long long>(w.b * p.Hq + head) * p.acc_rows + qrow;
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
        // The warp moves its 32 rows through its quarter of the slot's Q tile (no MMA reads it
        // any more: the unit's last S_s completed before its last P), CW columns at a time, so
        // that global loads and stores cover whole row segments: in a coalesced pass lane l
        // takes 16-byte chunk l % CPR of row l / CPR + RPI * i; in the row pass each thread
        // merges its own row. Chunk ch of row rr sits at rr * 4CW + 16 (ch ^ (rr & 7)) in the
        // stage. The first columns' old values are staged while the unit's last PV runs.
        constexpr int CW = D / 2;        // columns per pass: 32 rows x CW fp32 = a quarter tile
        constexpr int CPR = CW / 4;      // 16-byte fp32 chunks per row segment
        constexpr int RPI = 32 / CPR;    // rows per coalesced instruction
        constexpr int LPR = CW / 8;      // lanes per row segment of the bf16 copy
        const int qb = k & 1;
        uint8_t* stg = smem + C::OFF_Q + (qb * 2 + s) * C::TILE + qd * (32 * CW * 4);
        const long long wrow0 =
            static_cast<long long>(w.b * p.Hq + head) * p.acc_rows + q0s + qd * 32;
        const int wrows = min(32, p.Sq - (q0s + qd * 32));  // this warp's rows that exist
        const bool any_old = __any_sync(0xffffffffu, w_old != 0.f);
        auto sw = [](int rr, int ch) { return rr * (CW * 4) + ((ch ^ (rr & 7)) << 4); };
        auto stage_old = [&](int c0) {  // the old values of the warp's rows, into the stage
          // (some row exists here; the stage rows past the last one take copies of it)
          const float* abase = p.o_acc + wrow0 * D + c0;
#pragma unroll 1
          for (int i0 = 0; i0 < CPR; i0 += 8) {
            float4 a[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = min(RPI * (i0 + i) + lane / CPR, wrows - 1), ch = lane % CPR;
              a[i] = __ldcg(reinterpret_cast<const float4*>(abase + rr * D) + ch);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = RPI * (i0 + i) + lane / CPR, ch = lane % CPR;
              *reinterpret_cast<float4*>(stg + sw(rr, ch)) = a[i];
            }
          }
          __syncwarp();
        };
        if (any_old) stage_old(0);  // while the unit's last PV runs
        if (!wait_o()) {
          ok = false;
          break;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += CW) {
          float* const abase = p.o_acc + wrow0 * D + c0;  // row rr of the warp: abase + rr * D
          if (any_old && c0 > 0) stage_old(c0);
          // this thread's row, 32 columns at a time: O / l, plus the old values, into the stage
#pragma unroll 1
          for (int cb = 0; cb < CW; cb += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0 + cb, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4* sp = reinterpret_cast<float4*>(stg + sw(lane, cb / 4 + e));
              float4 v = make_float4(__uint_as_float(o[4 * e + 0]) * w_new,
                                     __uint_as_float(o[4 * e + 1]) * w_new,
                                     __uint_as_float(o[4 * e + 2]) * w_new,
                                     __uint_as_float(o[4 * e + 3]) * w_new);
              if (w_old != 0.f) {
                const float4 a = *sp;
                v.x += w_old * a.x;
                v.y += w_old * a.y;
                v.z += w_old * a.z;
                v.w += w_old * a.w;
              }
              *sp = v;
            }
          }
          __syncwarp();
          // the merged rows: fp32 into the accumulator, bf16 into out
#pragma unroll
          for (int i = 0; i < CPR; ++i) {
            const int rr = RPI * i + lane / CPR, ch = lane % CPR;
            if (rr < wrows)
              reinterpret_cast<float4*>(abase + rr * D)[ch] =
                  *reinterpret_cast<const float4*>(stg + sw(rr, ch));
          }
          if (p.out != nullptr) {
#pragma unroll
            for (int i = 0; i < LPR; ++i) {
              const int rr = (32 / LPR) * i + lane / LPR, c8 = lane % LPR;
              if (rr < wrows) {
                const float4 x0 = *reinterpret_cast<const float4*>(stg + sw(rr, 2 * c8));
                const float4 x1 = *reinterpret_cast<const float4*>(stg + sw(rr, 2 * c8 + 1));
                reinterpret_cast<uint4*>(p.out + (wrow0 + rr) * D + c0)[c8] =
                    make_uint4(pack_bf16(x0.x, x0.y), pack_bf16(x0.z, x0.w),
                               pack_bf16(x1.x, x1.y), pack_bf16(x1.z, x1.w));
              }
            }
          }
          __syncwarp();  // the stage is reused by the next columns
        }
        if (qrow < p.Sq) p.lse_acc[row] = lse_out;
        // this warp is done with the Q tile: the producer may reload the buffer
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_QSTAGED + qb));
      } else {
        if (!wait_o()) {
          ok = false;
          break;
        }
        // O / l -> bf16, written row by row into this slot's Q tile of the unit (no MMA reads
        // it any more: OFULL follows the unit's last S_s) in the 128-byte swizzled layout of
        // the output's tensor map; then one thread stores the tile with TMA (rows past Sq are
        // clipped by the map) and releases the buffer to the producer.
        const float inv = 1.0f / l;
        const int qb = k & 1;
        uint8_t* stage = smem + C::OFF_Q + (qb * 2 + s) * C::TILE;
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t o[32];
          tmem_ld32(tO + cb, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
            v.y = pack_bf16(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
            v.z = pack_bf16(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
            v.w = pack_bf16(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
            const int ch = (cb & 63) / 8 + e;  // 16-byte chunk within the 64-column block
            *reinterpret_cast<uint4*>(stage + (cb >> 6) * C::BLK + r * 128 + ((ch ^ (r & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::B_EPI + s));
        if (qd == 0 && lane == 0) {
          if (!mbar_wait(bar(C::B_EPI + s), k & 1, lim, abort_flag, p.status)) {
            ok = false;
          } else {
            if (w.q0 + slot_dq(p, s) < p.Sq)  // (the second tile of an odd count has no rows)
              for (int kb = 0; kb < C::KB; ++kb)
                tma_store_3d(&tm_o, smem_u32(stage + kb * C::BLK), kb * 64, w.q0 + slot_dq(p, s),
                             w.b * p.Hq + head);
            bulk_commit_group();
            bulk_wait_read_all();
            mbar_arrive(bar(C::B_QSTAGED + qb));
          }
        }
        __syncwarp();
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      // the next PFULL arrival (after tc_fence_before) orders these TMEM reads before the
      // next unit's first PV_s
    }
  }
  }
  // the output tiles stored with TMA have been written before the CTA exits
  if (warp >= 4 && (warp & 3) == 0 && lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace ra
