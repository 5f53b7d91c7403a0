// Split-KV decode attention over a pre-rotated KV cache (sm_100a), plus the log-sum-exp
// combine of the per-split partials.
//
// One decode step: the query of every head, at absolute position `pos`, is RoPE-rotated
// and attends the first L = min(Sk, pos+1) rows of an already-rotated key cache and the
// value cache ("Transformer internals: attention without the mysticism", "The KV cache and
// the memory wall": keys and values of past tokens are kept, and the step reads all of
// them; at batch 32 with an 8k context the cost is HBM traffic, not arithmetic).
//
// Work split: grid (n_splits, B * Hkv * hblocks). A CTA streams the K/V rows of one split
// of one KV head once from HBM (TMA, 128-byte swizzle, NST-deep ring of 64-key tiles) and
// serves up to 8 query heads of that KV group from it. Four consumer warps each take 16
// keys of every tile and compute with mma.sync m16n8k16 (bf16 -> fp32):
//   S^T[16 keys x 8 heads] = K_tile[16 x D] . q^T[D x 8]          (swap-AB: heads in N)
//   O^T[D x 8 heads]      += V^T[D x 16 keys] . P^T[16 keys x 8]    (V^T by ldmatrix.trans)
// P^T is turned from the accumulator layout into the B-operand layout with movmatrix.trans.
// Each warp keeps its own running max / sum per head (online softmax), the four warps are
// merged in shared memory, and the CTA writes one unnormalised partial (o, m, l) per head.
// decode_combine_kernel then merges the splits:
//   M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
//
// The same kernel serves every decode entry:
// * sequences at their own positions pos[b] (a varlen batch), each attending rows
//   lo_b .. pos_b with lo_b = pos_b - W + 1 under a sliding window W ("Building
//   Self-Attention and Transformer Engines" §6.4), else 0;
// * an optional append of the step's new token: the CTA whose key range holds row pos_b
//   rotates the new key to pos_b, stores it and the new value into the cache, and only then
//   loads its tiles, so the step attends its own token;
// * a contiguous cache [B, Hkv, S_cache, D] or a paged pool [num_blocks, Hkv, page, D]
//   reached through a block table (§6.2 PagedAttention), one TMA box per page.
// Key ranges are cut on 64-row boundaries of the absolute row index, so a tile is always
// whole pages. Rows of an edge tile outside [lo_b, L_b) are masked in S and their V rows
// are zeroed in shared memory before the PV product, so whatever those rows hold (stale
// cache contents, another sequence's page) cannot leak in, not even as NaN * 0.
#pragma once

#include "ptx.cuh"
#include "rope.cuh"

namespace ra {

struct DecParams {
  const __nv_bfloat16* q;  // [B, Hq, 1, D]
  float* part_o;           // [B * Hq, n_splits, D] unnormalised partial outputs
  float2* part_ml;         // [B * Hq, n_splits] (m, l), m in log2 units of the scaled score
  unsigned int* status;
  long long wait_limit;
  int B, Hq, Hkv, G;
  int cap;        // rows one sequence can hold: S_cache, or max_blocks * page
  int pos;        // position of every sequence when pos_arr is null
  const int* pos_arr;  // [B] per-sequence positions (device memory), or null
  int max_pos;    // bound on the positions the launch was sized for (checked)
  int window;     // 0 = no window; else keys pos-W+1 .. pos
  int n_splits;   // splits actually launched
  int chunk;      // keys per split (multiple of 64)
  int hblocks;    // ceil(G / 8): blocks of 8 query heads per KV head
  float scale_log2;
  float rope_base;
  // paged pool (page == 0: contiguous cache, maps over [B * Hkv, S_cache, D])
  int page;                // rows per page (divides 64)
  const int* block_table;  // [B, max_blocks]
  int max_blocks;
  int num_blocks;          // blocks in the pool (table entries are checked against it)
  // append of the step's token (k_new == null: none)
  const __nv_bfloat16* k_new;  // [B, Hkv, 1, D], not rotated
  const __nv_bfloat16* v_new;  // [B, Hkv, 1, D]
  __nv_bfloat16* k_cache;      // the memory tm_k covers
  __nv_bfloat16* v_cache;      // the memory tm_v covers
  int S_cache;
};

template <int D>
struct DecCfg {
  static constexpr int TK = 64;                 // keys per tile
  static constexpr int NDB = D / 64;            // 128-byte column blocks per row
  static constexpr int BOX = TK * 128;          // bytes of one 64-row column block
  static constexpr int TILE = TK * D * 2;       // bytes of one K (or V) tile
  static constexpr int STAGE = 2 * TILE;        // K tile then V tile
  static constexpr int NST = 3;
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_Q = NST * STAGE;                  // q_rot [8][D] bf16
  static constexpr int OFF_BAR = OFF_Q + 8 * D * 2;
  static constexpr int N_BAR = 2 * NST;
  static constexpr int OFF_ABORT = OFF_BAR + 8 * N_BAR;
  static constexpr int SMEM = OFF_ABORT + 16 + 1024;
  // merge scratch reuses the K/V ring once every tile has been consumed
  static constexpr int OFF_WS_O = 0;                         // [4 warps][8][D] fp32
  static constexpr int OFF_WS_ML = 4 * 8 * D * 4;            // [4 warps][8] float2
  static_assert(OFF_WS_ML + 4 * 8 * 8 <= NST * STAGE, "merge scratch");
};

// Byte offset of (key, d) inside one swizzled 64-key x D tile; d a multiple of 8. The tile is
// cut into groups of 2^lp keys (one page of a paged pool, or all 64 keys of a contiguous cache),
// each group holding its NDB 64-column blocks of 2^lp rows of 128 bytes: one TMA box per group
// fills it. The 128-byte swizzle moves 16-byte chunk c of a row to c ^ (key & 7).
template <int NDB, bool kPaged>
__device__ __forceinline__ uint32_t dec_swz(int key, int d, int lp) {
  if constexpr (!kPaged)  // one group of 64 keys: key < 64
    return static_cast<uint32_t>((d >> 6) * (64 * 128) + key * 128 +
                                 ((((d & 63) >> 3) ^ (key & 7)) << 4));
  const int grp = key >> lp, kin = key & ((1 << lp) - 1);
  return static_cast<uint32_t>(((((grp * NDB + (d >> 6)) << lp) + kin) << 7) +
                               ((((d & 63) >> 3) ^ (key & 7)) << 4));
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// kPaged: the cache is a paged pool (p.page > 0); the contiguous instance keeps the tile layout's
// key groups at their compile-time size of 64.
template <int D, bool kPaged>
__global__ void __launch_bounds__(160)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const DecParams p) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sKV = base + C::OFF_KV;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
  auto full = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * i; };
  auto empty = [&](int i) -> uint32_t { return base + C::OFF_BAR + 8u * (C::NST + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int hb = blockIdx.y % p.hblocks;
  const int kv_bh = blockIdx.y / p.hblocks;  // b * Hkv + kv head
  const int b = kv_bh / p.Hkv, g = kv_bh % p.Hkv;
  // this sequence's rows lo .. L-1; the launch covers rows (lo & ~63) + [0, n_splits * chunk)
  const int pos_b = p.pos_arr ? p.pos_arr[b] : p.pos;
  const int lo = (p.window > 0) ? max(0, pos_b - p.window + 1) : 0;
  const int L0 = min(p.cap, pos_b + 1);
  // (only the scalar-position contiguous call may name a position past the cache's end:
  // it then attends the whole cache)
  const bool strict = p.pos_arr != nullptr || p.page != 0 || p.k_new != nullptr;
  const bool bad = pos_b < 0 || pos_b > p.max_pos || (strict && pos_b >= p.cap) ||
                   L0 - (lo & ~63) > p.n_splits * p.chunk;
  const int L = bad ? 0 : L0;
  const int kstart = (lo & ~63) + split * p.chunk;
  const int kend = min(L, kstart + p.chunk);
  const int klo = max(lo, kstart);
  const int n_tiles = kend > klo ? (kend - kstart + C::TK - 1) / C::TK : 0;
  if (bad && threadIdx.x == 0 && split == 0 && hb == 0) atomicOr(p.status, kStatusArg);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------------- append + TMA producer
    if (p.k_new != nullptr && n_tiles > 0 && pos_b >= kstart && pos_b < kend) {
      // the step's own token: key rotated to pos_b, stored with its value at row pos_b,
      // ordered before this CTA's tile loads (async proxy) by the fence below
      long long row = -1;
      if (p.page == 0) {
        row = static_cast<long long>(kv_bh) * p.S_cache + pos_b;
      } else {
        const int blk = p.block_table[static_cast<long long>(b) * p.max_blocks + pos_b / p.page];
        if (blk >= 0 && blk < p.num_blocks)
          row = (static_cast<long long>(blk) * p.Hkv + g) * p.page + pos_b % p.page;
        else if (lane == 0)
          atomicOr(p.status, kStatusArg);
      }
      if (row >= 0) {
        const double log2_base = log2(static_cast<double>(p.rope_base));
        const uint4* kn = reinterpret_cast<const uint4*>(p.k_new + static_cast<long long>(kv_bh) * D);
        const uint4* vn = reinterpret_cast<const uint4*>(p.v_new + static_cast<long long>(kv_bh) * D);
        uint4* kd = reinterpret_cast<uint4*>(p.k_cache + row * D);
        uint4* vd = reinterpret_cast<uint4*>(p.v_cache + row * D);
        for (int c8 = lane; c8 < D / 8; c8 += 32) {
          float2 cs[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) rope_cos_sin(pos_b, c8 * 4 + t, D, log2_base, cs[t].x, cs[t].y);
          kd[c8] = rotate8(kn[c8], cs);
          vd[c8] = vn[c8];
        }
        fence_proxy_async_global();
      }
      __syncwarp();
    }
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      // The cache is read once: its lines go first when L2 needs room, so the stream replaces
      // its own lines rather than dirty lines that earlier kernels left (their write-back waits
      // for a kernel with DRAM to spare)
      const uint64_t pol = l2_policy_evict_first();
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % C::NST;
        if (t >= C::NST &&
            !mbar_wait(empty(st), ((t / C::NST) & 1) ^ 1, p.wait_limit, abort_flag, p.status))
          break;
        mbar_expect_tx(full(st), C::STAGE);
        const int key0 = kstart + t * C::TK;
        const uint32_t dst = sKV + st * C::STAGE;
        if (p.page == 0) {
#pragma unroll
          for (int db = 0; db < C::NDB; ++db) {
            tma_load_3d_hint(dst + db * C::BOX, &tm_k, db * 64, key0, kv_bh, full(st), pol);
            tma_load_3d_hint(dst + C::TILE + db * C::BOX, &tm_v, db * 64, key0, kv_bh, full(st),
                             pol);
          }
        } else {
          // one box per page; a page wholly outside [lo, L) loads the page of row pos_b in
          // its place (its rows are masked and its V rows zeroed by the consumers)
          for (int r0 = key0; r0 < key0 + C::TK; r0 += p.page) {
            const int rr = (r0 + p.page <= lo || r0 >= L) ? pos_b : r0;
            int blk = p.block_table[static_cast<long long>(b) * p.max_blocks + rr / p.page];
            if (blk < 0 || blk >= p.num_blocks) blk = p.num_blocks;  // past the map: zeros
            const int z = blk * p.Hkv + g;
            // the page's group: its column blocks one after the other (one box)
            const uint32_t o = static_cast<uint32_t>((r0 - key0) * 128 * C::NDB);
            if constexpr (C::NDB == 2) {
              tma_load_4d_hint(dst + o, &tm_k, 0, 0, 0, z, full(st), pol);
              tma_load_4d_hint(dst + C::TILE + o, &tm_v, 0, 0, 0, z, full(st), pol);
            } else {
              tma_load_3d_hint(dst + o, &tm_k, 0, 0, z, full(st), pol);
              tma_load_3d_hint(dst + C::TILE + o, &tm_v, 0, 0, z, full(st), pol);
            }
          }
        }
        issued = t + 1;
      }
      if (*abort_flag) {
        for (int t = max(0, issued - C::NST); t < issued; ++t)
          mbar_drain(full(t % C::NST), (t / C::NST) & 1);
      }
    }
    return;  // the producer takes no part in the consumers' named barriers
  }

  // ------------------------------------------------------------------ consumers
  const int cw = warp - 1;  // 0..3
  const int ct = threadIdx.x - 32;
  const int r = lane >> 2, c = lane & 3;
  __nv_bfloat16* q_rot = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_Q);

  // rotate the block's (up to) 8 query rows at `pos`; rows past G are zero
  {
    const double log2_base = log2(static_cast<double>(p.rope_base));
    for (int e = ct; e < 8 * (D / 2); e += 128) {
      const int hh = e / (D / 2), i = e % (D / 2);
      const int gh = hb * 8 + hh;
      float y0 = 0.f, y1 = 0.f;
      if (gh < p.G) {
        const __nv_bfloat16* qv = p.q + (static_cast<long long>(b) * p.Hq + g * p.G + gh) * D;
        const float x0 = __bfloat162float(qv[2 * i]), x1 = __bfloat162float(qv[2 * i + 1]);
        float cs, sn;
        rope_cos_sin(pos_b, i, D, log2_base, cs, sn);
        y0 = x0 * cs - x1 * sn;
        y1 = x0 * sn + x1 * cs;
      }
      q_rot[hh * D + 2 * i] = __float2bfloat16_rn(y0);
      q_rot[hh * D + 2 * i + 1] = __float2bfloat16_rn(y1);
    }
  }
  named_bar_sync(1, 128);
  uint32_t qf[D / 16][2];  // B fragments of q^T: (d = 16ks + 2c (+8), head r)
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qf[ks][0] = *reinterpret_cast<const uint32_t*>(q_rot + r * D + 16 * ks + 2 * c);
    qf[ks][1] = *reinterpret_cast<const uint32_t*>(q_rot + r * D + 16 * ks + 8 + 2 * c);
  }

  float acc[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2c, 2c+1
  const float sl2 = p.scale_log2;
  const int mi = lane >> 3, rr = lane & 7;
  const int krow = cw * 16;
  const int lp = kPaged ? __ffs(p.page) - 1 : 6;  // log2 of the keys per TMA group

  bool ok = true;
  for (int t = 0; t < n_tiles; ++t) {
    const int st = t % C::NST;
    if (!mbar_wait_warp(full(st), (t / C::NST) & 1, p.wait_limit, abort_flag, p.status)) {
      ok = false;
      break;
    }
    const uint32_t kS = sKV + st * C::STAGE, vS = kS + C::TILE;
    const int tile0 = kstart + t * C::TK;
    const bool edge = tile0 < klo || tile0 + C::TK > kend;
    if (edge) {
      // zero the V rows of this warp's keys outside [klo, kend): P is 0 there, but 0 * NaN
      // is not
      for (int idx = lane; idx < 16 * (D / 8); idx += 32) {
        const int i = idx / (D / 8), c8 = idx % (D / 8);
        const int kk = tile0 + krow + i;
        if (kk < klo || kk >= kend) st_shared_zero16(vS + dec_swz<C::NDB, kPaged>(krow + i, 8 * c8, lp));
      }
      __syncwarp();
    }

    // S^T = K . q^T over this warp's 16 keys
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(kS + dec_swz<C::NDB, kPaged>(krow + (mi & 1) * 8 + rr, 16 * ks + (mi >> 1) * 8, lp), a0, a1,
              a2, a3);
      mma_bf16_16816(sc, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
    }
    // sc[0]/[1]: key krow+r, heads 2c/2c+1; sc[2]/[3]: key krow+r+8
    const int kg = tile0 + krow + r;
    float x0 = sc[0] * sl2, x1 = sc[1] * sl2, x2 = sc[2] * sl2, x3 = sc[3] * sl2;
    if (kg >= kend || kg < klo) x0 = x1 = -INFINITY;
    if (kg + 8 >= kend || kg + 8 < klo) x2 = x3 = -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const bool e0 = mn0 == -INFINITY, e1 = mn1 == -INFINITY;  // nothing seen yet
    const float al0 = e0 ? 1.f : ex2(m0 - mn0), al1 = e1 ? 1.f : ex2(m1 - mn1);
    const float p0 = e0 ? 0.f : ex2(x0 - mn0), p2 = e0 ? 0.f : ex2(x2 - mn0);
    const float p1 = e1 ? 0.f : ex2(x1 - mn1), p3 = e1 ? 0.f : ex2(x3 - mn1);
    l0 = l0 * al0 + p0 + p2;
    l1 = l1 * al1 + p1 + p3;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      acc[mt][0] *= al0;
      acc[mt][1] *= al1;
      acc[mt][2] *= al0;
      acc[mt][3] *= al1;
    }
    // P^T as the B operand: (keys 2c,2c+1 ; head r) for keys 0-7 and 8-15
    const uint32_t b0 = movmatrix_t(pack_bf16(p0, p1));
    const uint32_t b1 = movmatrix_t(pack_bf16(p2, p3));
    // O^T += V^T . P^T
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(vS + dec_swz<C::NDB, kPaged>(krow + (mi >> 1) * 8 + rr, 16 * mt + (mi & 1) * 8, lp), a0,
                a1, a2, a3);
      mma_bf16_16816(acc[mt], a0, a1, a2, a3, b0, b1);
    }
    if (edge) fence_proxy_async_smem();  // the generic zeroing before the next TMA fill
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
  }

  // every tile is consumed: the combine kernel may be scheduled now (its CTAs wait in
  // grid_dep_wait until this grid has completed and written its partials)
  grid_dep_launch();
  // reduce the per-lane sums over the 8 lanes that share a head column
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  // all consumer warps are done with the ring before it becomes merge scratch
  named_bar_sync(1, 128);
  float* ws_o = reinterpret_cast<float*>(smem + C::OFF_KV + C::OFF_WS_O);
  float2* ws_ml = reinterpret_cast<float2*>(smem + C::OFF_KV + C::OFF_WS_ML);
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const int d = 16 * mt + r;
    ws_o[(cw * 8 + 2 * c) * D + d] = acc[mt][0];
    ws_o[(cw * 8 + 2 * c + 1) * D + d] = acc[mt][1];
    ws_o[(cw * 8 + 2 * c) * D + d + 8] = acc[mt][2];
    ws_o[(cw * 8 + 2 * c + 1) * D + d + 8] = acc[mt][3];
  }
  if (r == 0) {
    ws_ml[cw * 8 + 2 * c] = make_float2(m0, l0);
    ws_ml[cw * 8 + 2 * c + 1] = make_float2(m1, l1);
  }
  named_bar_sync(1, 128);
  if (!ok || *abort_flag) return;

  // merge the four warps; write this split's partial per head
  const int nh = min(8, p.G - hb * 8);
  for (int e = ct; e < nh * D; e += 128) {
    const int hh = e / D, d = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, ws_ml[w * 8 + hh].x);
    float o = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float2 ml = ws_ml[w * 8 + hh];
      const float f = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M);
      o += f * ws_o[(w * 8 + hh) * D + d];
      l += f * ml.y;
    }
    const long long row = (static_cast<long long>(b) * p.Hq + g * p.G + hb * 8 + hh) * p.n_splits + split;
    p.part_o[row * D + d] = o;
    if (d == 0) p.part_ml[row] = make_float2(M, l);
  }
}

// the merge of the splits: out[b, h, 0, :] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
// Launched right behind the split kernel with a programmatic dependency, so its launch
// overlaps the split kernel's last wave; it reads the partials only after grid_dep_wait.
__global__ void decode_combine_kernel(const float* __restrict__ part_o,
                                      const float2* __restrict__ part_ml,
                                      __nv_bfloat16* __restrict__ out, int n_splits, int D) {
  grid_dep_wait();
  const long long bh = blockIdx.x;
  const float2* ml = part_ml + bh * n_splits;
  float M = -INFINITY;
  for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ml[s].x);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float o = 0.f, l = 0.f;
    for (int s = 0; s < n_splits; ++s) {
      const float2 v = ml[s];
      const float f = (v.x == -INFINITY) ? 0.f : ex2(v.x - M);
      o += f * part_o[(bh * n_splits + s) * D + d];
      l += f * v.y;
    }
    out[bh * D + d] = __float2bfloat16_rn(o / l);
  }
}

}  // namespace ra
