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
// Q is rotated in shared memory by its softmax group right after the TMA load (a3); K is
// rotated once per call by rope_rotate_kernel into a workspace (a2), since every K tile is
// re-read by S/128 query tiles.
#pragma once

#include "ptx.cuh"
#include "rope.cuh"

namespace ra {

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
  int q_tab_off;        // table row of query row 0
  float scale_log2;     // log2(e) / sqrt(D)
};

template <int D>
struct FwdCfg {
  static constexpr int KB = D / 64;                  // 128-byte column blocks per row
  static constexpr int BLK = 128 * 128;              // bytes of one 128-row column block
  static constexpr int TILE = 128 * D * 2;           // bytes of one 128 x D bf16 tile
  static constexpr int NST = (D == 128) ? 2 : 4;     // K/V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + NST * TILE;
  static constexpr int OFF_BAR = OFF_V + NST * TILE;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;  // barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  // TMEM columns: S/P of slot s at 128*s, O of slot s at 256 + D*s
  __device__ static constexpr uint32_t col_s(int s) { return 128u * static_cast<uint32_t>(s); }
  __device__ static constexpr uint32_t col_o(int s) { return 256u + static_cast<uint32_t>(D * s); }
  // barrier indices (8 bytes each)
  static constexpr int B_QFULL = 0, B_QREADY = 2, B_SFULL = 4, B_PFULL = 6, B_OFULL = 8,
                       B_DRAIN = 10, B_KFULL = 11, B_KEMPTY = 11 + NST, B_VFULL = 11 + 2 * NST,
                       B_VEMPTY = 11 + 3 * NST, N_BAR = 11 + 4 * NST;
  static constexpr int OFF_TMEM_SLOT = 8 * N_BAR;
  static constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
  static_assert(OFF_ABORT + 4 <= 512, "barrier area");
};

template <int D>
__global__ void __launch_bounds__(384, 1)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q, sK = base + C::OFF_K, sV = base + C::OFF_V;
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
  const int off = p.Sk - p.Sq;  // query row i sits at key index i + off
  int n_kv = (p.Sk + 127) / 128;
  if (p.causal) n_kv = min(n_kv, (min(p.Sq - 1, q0 + 127) + off) / 128 + 1);
  const int ns = p.n_slots;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::B_QFULL + s), 1);
      mbar_init(bar(C::B_QREADY + s), 128);
      mbar_init(bar(C::B_SFULL + s), 1);
      mbar_init(bar(C::B_PFULL + s), 128);
      mbar_init(bar(C::B_OFULL + s), 1);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(bar(C::B_KFULL + i), 1);
      mbar_init(bar(C::B_KEMPTY + i), 1);
      mbar_init(bar(C::B_VFULL + i), 1);
      mbar_init(bar(C::B_VEMPTY + i), 1);
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
  // warpgroup gives back to 56, the two softmax warpgroups take 224
  // (128 x 56 + 256 x 224 = 64512).
  if (warp < 4) {
  regs_dec<56>();
  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int s = 0; s < ns; ++s) {
        mbar_expect_tx(bar(C::B_QFULL + s), C::TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(sQ + s * C::TILE + kb * C::BLK, &tm_q, kb * 64, q0, b * p.Hq + h0 + s,
                      bar(C::B_QFULL + s));
      }
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::NST;
        const uint32_t ph = (j / C::NST) & 1;
        if (j >= C::NST &&
            !mbar_wait(bar(C::B_KEMPTY + st), ph ^ 1, p.wait_limit, abort_flag, p.status))
          break;
        mbar_expect_tx(bar(C::B_KFULL + st), C::TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(sK + st * C::TILE + kb * C::BLK, &tm_k, kb * 64, j * 128, kv_bh,
                      bar(C::B_KFULL + st));
        if (j >= C::NST &&
            !mbar_wait(bar(C::B_VEMPTY + st), ph ^ 1, p.wait_limit, abort_flag, p.status)) {
          issued = -(j + 1);  // K of tile j in flight, V not
          break;
        }
        mbar_expect_tx(bar(C::B_VFULL + st), C::TILE);
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_3d(sV + st * C::TILE + kb * C::BLK, &tm_v, kb * 64, j * 128, kv_bh,
                      bar(C::B_VFULL + st));
        issued = j + 1;
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA can exit
        for (int s = 0; s < ns; ++s) mbar_drain(bar(C::B_QFULL + s), 0);
        const int nk = issued >= 0 ? issued : -issued;
        const int nv = issued >= 0 ? issued : -issued - 1;
        for (int j = max(0, nk - C::NST); j < nk; ++j)
          mbar_drain(bar(C::B_KFULL + j % C::NST), (j / C::NST) & 1);
        for (int j = max(0, nv - C::NST); j < nv; ++j)
          mbar_drain(bar(C::B_VFULL + j % C::NST), (j / C::NST) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = umma_idesc_bf16(128, 128, 0, 0);  // Q, K both K-major
      constexpr uint32_t kIdescO = umma_idesc_bf16(128, D, 0, 1);    // V is MN-major
      auto issue_s = [&](int s, int st) {
        const uint32_t d_t = tmem + C::col_s(s);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t o = (k >> 2) * C::BLK + (k & 3) * 32;
          const uint64_t ad = umma_smem_desc(sQ + s * C::TILE + o, 16, 1024, kLayoutSW128);
          const uint64_t bd = umma_smem_desc(sK + st * C::TILE + o, 16, 1024, kLayoutSW128);
          umma_ss(d_t, ad, bd, kIdescS, k > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int s, int st, bool acc) {
        const uint32_t d_t = tmem + C::col_o(s);
        const uint32_t a_t = tmem + C::col_s(s);
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // 128 keys, 16 per MMA
          const uint64_t bd =
              umma_smem_desc(sV + st * C::TILE + k * 2048, C::BLK, 1024, kLayoutSW128);
          umma_ts(d_t, a_t + 8 * k, bd, kIdescO, (acc || k > 0) ? 1u : 0u);
        }
      };
      const long long lim = p.wait_limit;
      bool ok = mbar_wait(bar(C::B_QREADY + 0), 0, lim, abort_flag, p.status) &&
                mbar_wait(bar(C::B_KFULL + 0), 0, lim, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        umma_commit(bar(C::B_SFULL + 0));
        if (ns == 2) {
          ok = mbar_wait(bar(C::B_QREADY + 1), 0, lim, abort_flag, p.status);
          if (ok) {
            tc_fence_after();
            issue_s(1, 0);
            umma_commit(bar(C::B_SFULL + 1));
          }
        }
        umma_commit(bar(C::B_KEMPTY + 0));
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % C::NST;
        const uint32_t ph = (j / C::NST) & 1;
        const bool has_next = j + 1 < n_kv;
        const int st1 = (j + 1) % C::NST;
        const uint32_t ph1 = ((j + 1) / C::NST) & 1;
        if (!mbar_wait(bar(C::B_PFULL + 0), j & 1, lim, abort_flag, p.status) ||
            !mbar_wait(bar(C::B_VFULL + st), ph, lim, abort_flag, p.status))
          break;
        tc_fence_after();
        issue_pv(0, st, j > 0);
        if (!has_next) umma_commit(bar(C::B_OFULL + 0));
        if (has_next) {
          if (!mbar_wait(bar(C::B_KFULL + st1), ph1, lim, abort_flag, p.status)) break;
          tc_fence_after();
          issue_s(0, st1);
          umma_commit(bar(C::B_SFULL + 0));
        }
        if (ns == 2) {
          if (!mbar_wait(bar(C::B_PFULL + 1), j & 1, lim, abort_flag, p.status)) break;
          tc_fence_after();
          issue_pv(1, st, j > 0);
          if (!has_next) umma_commit(bar(C::B_OFULL + 1));
          umma_commit(bar(C::B_VEMPTY + st));
          if (has_next) {
            issue_s(1, st1);
            umma_commit(bar(C::B_SFULL + 1));
            umma_commit(bar(C::B_KEMPTY + st1));
          }
        } else {
          umma_commit(bar(C::B_VEMPTY + st));
          if (has_next) umma_commit(bar(C::B_KEMPTY + st1));
        }
      }
      // every MMA issued above must finish before TMEM is released
      umma_commit(bar(C::B_DRAIN));
      mbar_drain(bar(C::B_DRAIN), 0);
    }
    __syncwarp();
  }
  } else {
  regs_inc<224>();
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

    // a3: rotate this row of Q_s in shared memory (128-byte swizzled layout of the TMA box)
    bool ok = mbar_wait_warp(bar(C::B_QFULL + s), 0, lim, abort_flag, p.status);
    if (ok && qrow < p.Sq) {
      const float4* trow = reinterpret_cast<const float4*>(
          p.tab + static_cast<long long>(p.q_tab_off + qrow) * (D / 2));
      uint8_t* qrow_base = smem + C::OFF_Q + s * C::TILE + r * 128;
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(qrow_base + kb * C::BLK + ((c ^ (r & 7)) << 4));
          const int pair0 = kb * 32 + c * 4;
          const float4 a = __ldg(trow + pair0 / 2), bq = __ldg(trow + pair0 / 2 + 1);
          const float2 cs[4] = {make_float2(a.x, a.y), make_float2(a.z, a.w),
                                make_float2(bq.x, bq.y), make_float2(bq.z, bq.w)};
          *ptr = rotate8(*ptr, cs);
        }
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(bar(C::B_QREADY + s));

    float m = -INFINITY;  // running row max, in log2 units of the scaled score
    float l = 0.f;        // running row sum of 2^(x - m)
    const float sl2 = p.scale_log2;
    const int lim_causal = min(p.Sk - 1, qrow + off);
    for (int j = 0; ok && j < n_kv; ++j) {
      if (!mbar_wait_warp(bar(C::B_SFULL + s), j & 1, lim, abort_flag, p.status)) {
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

      // a6: causal / sequence-end mask, only on tiles that reach past some row's limit
      const int kbase = j * 128;
      const bool need_mask = (kbase + 128 > p.Sk) || (p.causal && kbase + 127 > q0 + off);
      if (need_mask) {
        const int lim_k = (p.causal ? lim_causal : p.Sk - 1) - kbase;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim_k) sr[c] = 0xff800000u;  // -inf
      }
      // a7: online softmax with a lazily updated reference max
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mt = fmaxf(mt, __uint_as_float(sr[c]));
      const float m_new = fmaxf(m, mt * sl2);
      // Keep the old reference unless the max grew by more than 8 (P stays <= 256);
      // O / l is exact for any common reference, so skipping the rescale is lossless.
      const bool upd = m_new > m + 8.0f;
      const float alpha = upd ? ex2(m - m_new) : 1.0f;
      if (upd) m = m_new;
      l *= alpha;
      if (j > 0 && __any_sync(0xffffffffu, upd)) {
        // a8: O_s *= alpha (PV_s(j-1) has completed: it was issued before S_s(j))
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
      const float neg_m = -m;
      float rs = 0.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) {
          const int c = h * 64 + 2 * c2;
          const float p0 = ex2(fmaf(__uint_as_float(sr[c]), sl2, neg_m));
          const float p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), sl2, neg_m));
          rs += p0 + p1;
          pk[c2] = pack_bf16(p0, p1);
        }
        tmem_st32(tS + 32 * h, pk);
      }
      l += rs;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::B_PFULL + s));
    }

    // a10: epilogue O / l -> bf16
    if (ok && mbar_wait_warp(bar(C::B_OFULL + s), 0, lim, abort_flag, p.status)) {
      tc_fence_after();
      const float inv = 1.0f / l;
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
            dst[i] = w;
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
