// RoPE on sm_100a: the rotation angles and the HBM-bound rotation of whole K (or any
// [rows, S, D] bf16 tensor).
//
// Rotary Position Embeddings as in "Transformer Architecture & Self-Attention
// Mechanics" (devthesis.com), §3 "Rotary Position Embeddings (RoPE)": the pair
// (x_2i, x_2i+1) of a row at absolute position m is multiplied by
// [[cos m*theta_i, -sin m*theta_i], [sin m*theta_i, cos m*theta_i]] with
// theta_i = base^(-2i/D); the base is a parameter ("Transformer internals: attention
// without the mysticism", section "Rotary positional embeddings (RoPE)").
//
// Angles reach 32767 rad at S = 32768, where a float product alone is off by ~2e-3
// rad, so theta_i and m*theta_i are formed in fp64 and cos/sin taken in fp64 before
// narrowing to fp32.
#pragma once

#include "ptx.cuh"

namespace ra {

__device__ __forceinline__ void rope_cos_sin(long long pos, int i, int D, double log2_base,
                                             float& c, float& s) {
  const double theta = exp2(-(2.0 * i / D) * log2_base);  // base^(-2i/D)
  double sd, cd;
  sincos(static_cast<double>(pos) * theta, &sd, &cd);
  c = static_cast<float>(cd);
  s = static_cast<float>(sd);
}

// Table of (cos, sin) for `rows` consecutive absolute positions starting at pos0:
// tab[r * D/2 + i] = (cos, sin)((pos0 + r) * theta_i).
__global__ void rope_table_kernel(float2* __restrict__ tab, long long pos0, int rows, int D,
                                  float base) {
  const double log2_base = log2(static_cast<double>(base));
  const long long n = static_cast<long long>(rows) * (D / 2);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = static_cast<int>(e / (D / 2));
    const int i = static_cast<int>(e % (D / 2));
    float c, s;
    rope_cos_sin(pos0 + r, i, D, log2_base, c, s);
    tab[e] = make_float2(c, s);
  }
}

// Rotate 8 bf16 (4 pairs) given their 4 (cos, sin) pairs; fp32 math, bf16 RNE store.
__device__ __forceinline__ uint4 rotate8(uint4 x, const float2 (&cs)[4]) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const float x0 = bf16_lo(w[t]), x1 = bf16_hi(w[t]);
    o[t] = pack_bf16(x0 * cs[t].x - x1 * cs[t].y, x0 * cs[t].y + x1 * cs[t].x);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The two elementwise kernels below walk tiles of (kRotHeads heads) x (256 / (D/8) rows): a
// block of 256 threads takes one tile per pass, thread t the 16-byte chunk t % (D/8) of row
// t / (D/8) in each of the tile's heads; when D/8 does not divide 256, the threads past the
// tile's last whole row idle. Each thread reads (or forms) its angles once and has its
// kRotHeads loads in flight together before the first store. Grids are sized by rope_tiles
// and stride over the tiles.
constexpr int kRotHeads = 8;
constexpr int kRotThreads = 256;

__host__ __device__ inline int rope_rows_per_tile(int D) { return kRotThreads / (D / 8); }

// Tiles over `heads` heads of S rows.
__host__ __device__ inline long long rope_tiles(long long heads, int S, int D) {
  const int rpt = rope_rows_per_tile(D);
  return (heads + kRotHeads - 1) / kRotHeads * ((S + rpt - 1) / rpt);
}

// (cos, sin) of the 4 pairs of 16-byte chunk `chunk` at table row `row`.
__device__ __forceinline__ void table_cs(const float2* __restrict__ tab, long long row, int chunk,
                                         int D, float2 (&cs)[4]) {
  const float4* t4 = reinterpret_cast<const float4*>(tab + row * (D / 2) + chunk * 4);
  const float4 a = __ldg(t4), b = __ldg(t4 + 1);
  cs[0] = make_float2(a.x, a.y);
  cs[1] = make_float2(a.z, a.w);
  cs[2] = make_float2(b.x, b.y);
  cs[3] = make_float2(b.z, b.w);
}

// x, y: `heads` = nrows_total / S heads of S rows of D bf16; row s of head h at h * x_rows + s
// (x) and h * y_rows + s (y); rows sit at sequence index s.
// kTable: angles from `tab` (row tab_off + s); else computed here at pos0 + s.
// In place (x == y, x_rows == y_rows) is allowed: each thread reads its chunks before it
// writes them.
template <bool kTable>
__global__ void __launch_bounds__(kRotThreads) rope_rotate_kernel(const uint4* x, uint4* y,
                                                                  const float2* __restrict__ tab,
                                                                  long long nrows_total, int S,
                                                                  int D, long long pos0,
                                                                  int tab_off, float base,
                                                                  int x_rows, int y_rows) {
  const int cpr = D / 8;  // 16-byte chunks per row
  const int rpt = rope_rows_per_tile(D);
  const int chunk = threadIdx.x % cpr, r_in = threadIdx.x / cpr;
  if (r_in >= rpt) return;  // past the tile's last whole row: that row is the next tile's
  const int heads = static_cast<int>(nrows_total / S);
  const int row_tiles = (S + rpt - 1) / rpt;
  const int n_tiles = (heads + kRotHeads - 1) / kRotHeads * row_tiles;
  const double log2_base = kTable ? 0.0 : log2(static_cast<double>(base));
  for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int g = t / row_tiles;
    const int s = (t - g * row_tiles) * rpt + r_in;
    if (s >= S) continue;
    const int h0 = g * kRotHeads;
    const int nh = min(kRotHeads, heads - h0);
    uint4 v[kRotHeads];
#pragma unroll
    for (int h = 0; h < kRotHeads; ++h)
      if (h < nh) v[h] = x[(static_cast<long long>(h0 + h) * x_rows + s) * cpr + chunk];
    float2 cs[4];
    if (kTable) {
      table_cs(tab, tab_off + s, chunk, D, cs);
    } else {
#pragma unroll
      for (int t4 = 0; t4 < 4; ++t4)
        rope_cos_sin(pos0 + s, chunk * 4 + t4, D, log2_base, cs[t4].x, cs[t4].y);
    }
#pragma unroll
    for (int h = 0; h < kRotHeads; ++h)
      if (h < nh) y[(static_cast<long long>(h0 + h) * y_rows + s) * cpr + chunk] = rotate8(v[h], cs);
  }
}

// Prefill into a KV cache: the chunk's keys k [BH, S, D] are rotated (angles from table row
// tab_off + s, i.e. position pos0 + s) into rows pos0 + s of each [S_cache, D] slice of kc,
// and the values v are copied to the same rows of vc. One pass over the chunk.
__global__ void __launch_bounds__(kRotThreads) cache_write_kernel(const uint4* __restrict__ k,
                                                                  const uint4* __restrict__ v,
                                                                  uint4* __restrict__ kc,
                                                                  uint4* __restrict__ vc,
                                                                  const float2* __restrict__ tab,
                                                                  long long bh_count, int S,
                                                                  int S_cache, int pos0, int D,
                                                                  int tab_off) {
  const int cpr = D / 8;
  const int rpt = rope_rows_per_tile(D);
  const int chunk = threadIdx.x % cpr, r_in = threadIdx.x / cpr;
  if (r_in >= rpt) return;
  const int heads = static_cast<int>(bh_count);
  const int row_tiles = (S + rpt - 1) / rpt;
  const int n_tiles = (heads + kRotHeads - 1) / kRotHeads * row_tiles;
  for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int g = t / row_tiles;
    const int s = (t - g * row_tiles) * rpt + r_in;
    if (s >= S) continue;
    const int h0 = g * kRotHeads;
    const int nh = min(kRotHeads, heads - h0);
    uint4 kv[kRotHeads], vv[kRotHeads];
#pragma unroll
    for (int h = 0; h < kRotHeads; ++h) {
      if (h < nh) {
        const long long src = (static_cast<long long>(h0 + h) * S + s) * cpr + chunk;
        kv[h] = __ldg(k + src);
        vv[h] = __ldg(v + src);
      }
    }
    float2 cs[4];
    table_cs(tab, tab_off + s, chunk, D, cs);
#pragma unroll
    for (int h = 0; h < kRotHeads; ++h) {
      if (h < nh) {
        const long long dst = (static_cast<long long>(h0 + h) * S_cache + pos0 + s) * cpr + chunk;
        kc[dst] = rotate8(kv[h], cs);
        vc[dst] = vv[h];
      }
    }
  }
}

}  // namespace ra
