// k_reorder_pool.cu -- token reordering and hierarchical mean pooling.
//
// Both are pure HBM streams: every token row (d elements, 128 B for bf16 at
// d = 64) is read once and written once, moved as 16-byte vectors so that a
// warp touches whole 32-byte sectors.
#include "llsa_internal.cuh"

namespace llsa {

// Hierarchical position of pixel (y, x): recursive t x t tiles, row-major in
// every tile and across the top grid of t^L x t^L squares (index reordering of
// the Trainable Log-linear Sparse Attention summary, §4.2 / Fig. 2).
__device__ __forceinline__ int64_t hier_index(int64_t y, int64_t x, int t, int L, int W, int64_t BL) {
  int64_t tL = 1;
  for (int l = 0; l < L; ++l) tL *= t;
  int64_t h = ((y / tL) * (W / tL) + x / tL) * BL;
  int64_t Bp = 1;
  for (int l = 1; l <= L; ++l) {
    h += ((y % t) * t + (x % t)) * Bp;
    y /= t;
    x /= t;
    Bp *= (int64_t)t * t;
  }
  return h;
}

// One thread per 16-byte vector of a token row; consecutive threads walk a
// raster row, so the raster side is read or written fully coalesced and the
// hierarchical side moves whole rows.
__global__ void reorder_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int64_t rows_per_slice,
                               int vec_per_row, int64_t total, int t, int L, int W, int64_t BL, int to_hier) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t row = e / vec_per_row;
    int vcol = (int)(e - row * vec_per_row);
    int64_t bh = row / rows_per_slice;
    int64_t r = row - bh * rows_per_slice;          // raster position
    int64_t h = hier_index(r / W, r % W, t, L, W, BL);
    int64_t base = bh * rows_per_slice;
    if (to_hier)
      out[(base + h) * vec_per_row + vcol] = in[(base + r) * vec_per_row + vcol];
    else
      out[(base + r) * vec_per_row + vcol] = in[(base + h) * vec_per_row + vcol];
  }
}

// The same with 32-bit index arithmetic, for tile sides t = 2^lt and fewer
// than 2^32 vectors in all: per vector three 32-bit divisions and shifts, so
// that the copy stays bound by memory rather than by the index math.
__global__ void reorder32_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, uint32_t N, uint32_t vec,
                                 uint32_t total, int lt, int L, uint32_t W, uint32_t Gw, int to_hier) {
  const uint32_t tmask = (1u << lt) - 1u;
  const int ltL = lt * L;
  for (uint32_t e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
    const uint32_t row = e / vec, vcol = e - row * vec;
    const uint32_t bh = row / N, r = row - bh * N;         // raster position within the slice
    const uint32_t y = r / W, x = r - y * W;
    uint32_t h = ((y >> ltL) * Gw + (x >> ltL)) << (2 * ltL);
    for (int l = 0; l < L; ++l)
      h |= ((((y >> (lt * l)) & tmask) << lt) | ((x >> (lt * l)) & tmask)) << (2 * lt * l);
    const size_t base = (size_t)bh * N;
    const size_t rr = (base + r) * vec + vcol, hh = (base + h) * vec + vcol;
    if (to_hier)
      out[hh] = in[rr];
    else
      out[rr] = in[hh];
  }
}

static int grid_for(int64_t work, int threads) {
  int64_t blocks = (work + threads - 1) / threads;
  int64_t cap = 148ll * 16;
  return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

cudaError_t launch_reorder(const Geo& g, const void* in, void* out, int to_hier, cudaStream_t s) {
  int vec = g.d * (g.bf16 ? 2 : 4) / 16;
  int64_t total = (int64_t)g.BH * g.N * vec;
  int lt = 0;
  while ((1 << lt) < g.t) ++lt;
  if ((1 << lt) == g.t && total < (1ll << 32)) {
    int64_t tl = 1;
    for (int l = 0; l < g.L; ++l) tl *= g.t;
    reorder32_kernel<<<grid_for(total, 256), 256, 0, s>>>((const uint4*)in, (uint4*)out, (uint32_t)g.N,
                                                          (uint32_t)vec, (uint32_t)total, lt, g.L, (uint32_t)g.W,
                                                          (uint32_t)(g.W / tl), to_hier);
    note_launches(1);
    return cudaGetLastError();
  }
  reorder_kernel<<<grid_for(total, 256), 256, 0, s>>>((const uint4*)in, (uint4*)out, g.N, vec, total, g.t,
                                                      g.L, g.W, g.Bl[g.L], to_hier);
  note_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ pool

__device__ __forceinline__ void load4(const float* p, float* v) {
  float4 x = *reinterpret_cast<const float4*>(p);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* v) {
  uint2 x = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&x.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&x.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}

// Level l from level l-1: P_l[j] = (1/B) sum_{r<B} P_{l-1}[j*B + r]
// (hierarchical compression, Trainable Log-linear Sparse Attention summary §三).
// One thread per (slice, pooled token, 4 channels); fp32 accumulation in the
// order r = 0..B-1.  With B a compile-time constant all B row loads of a
// thread are in flight at once.
template <typename Tin, int BC>
__global__ void pool_level_kernel(const Tin* __restrict__ in, float* __restrict__ out, int d, int Brt,
                                  int64_t total) {
  const int B = BC > 0 ? BC : Brt;
  int c4n = d / 4;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t tok = e / c4n;                       // (slice, j) flattened: slices are consecutive
    int c = (int)(e - tok * c4n) * 4;
    const Tin* src = in + tok * B * d + c;       // rows j*B .. j*B+B-1 of the same slice
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (BC > 0) {
      float v[BC > 0 ? BC : 1][4];
#pragma unroll
      for (int r = 0; r < BC; ++r) load4(src + (int64_t)r * d, v[r]);
#pragma unroll
      for (int r = 0; r < BC; ++r) {
        acc[0] += v[r][0]; acc[1] += v[r][1]; acc[2] += v[r][2]; acc[3] += v[r][3];
      }
    } else {
      for (int r = 0; r < B; ++r) {
        float v[4];
        load4(src + (int64_t)r * d, v);
        acc[0] += v[0]; acc[1] += v[1]; acc[2] += v[2]; acc[3] += v[3];
      }
    }
    float4 o = make_float4(acc[0] / B, acc[1] / B, acc[2] / B, acc[3] / B);
    *reinterpret_cast<float4*>(out + tok * d + c) = o;
  }
}

template <typename Tin>
static void pool_launch(const Tin* in, float* out, const Geo& g, int64_t total, cudaStream_t s) {
  const int grid = grid_for(total, 256);
  if (g.B == 16)
    pool_level_kernel<Tin, 16><<<grid, 256, 0, s>>>(in, out, g.d, g.B, total);
  else if (g.B == 4)
    pool_level_kernel<Tin, 4><<<grid, 256, 0, s>>>(in, out, g.d, g.B, total);
  else
    pool_level_kernel<Tin, 0><<<grid, 256, 0, s>>>(in, out, g.d, g.B, total);
}

// Levels 1 and 2 in one pass for B = 16, d = 64: one CTA per level-2 token
// (256 fine rows).  Thread t sums the 16 rows of level-1 token t / 16 on
// channels 4 (t % 16) .. +3 in row order, divides by B (the same operations
// as pool_level_kernel), writes it and keeps it in shared memory; then 16
// threads sum the 16 level-1 values of each channel group in order for the
// level-2 token.  Lanes 0-15 of a warp read one 128-byte row, lanes 16-31 the
// next token's.
template <typename Tin>
__global__ void __launch_bounds__(256) pool_l12_kernel(const Tin* __restrict__ in, float* __restrict__ p1,
                                                       float* __restrict__ p2) {
  constexpr int B = 16, D = 64;
  __shared__ float4 lvl1[B][D / 4];
  const int t = threadIdx.x;
  const int j = t >> 4, c4 = (t & 15) * 4;
  const int64_t tok2 = blockIdx.x;                   // (slice, level-2 token) flattened
  const int64_t tok1 = tok2 * B + j;
  const Tin* src = in + tok1 * B * D + c4;
  float v[B][4];
#pragma unroll
  for (int r = 0; r < B; ++r) load4(src + (int64_t)r * D, v[r]);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int r = 0; r < B; ++r) {
    acc[0] += v[r][0]; acc[1] += v[r][1]; acc[2] += v[r][2]; acc[3] += v[r][3];
  }
  const float4 o = make_float4(acc[0] / B, acc[1] / B, acc[2] / B, acc[3] / B);
  *reinterpret_cast<float4*>(p1 + tok1 * D + c4) = o;
  lvl1[j][t & 15] = o;
  __syncthreads();
  if (t < D / 4) {
    float a2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < B; ++r) {
      const float4 w = lvl1[r][t];
      a2[0] += w.x; a2[1] += w.y; a2[2] += w.z; a2[3] += w.w;
    }
    *reinterpret_cast<float4*>(p2 + tok2 * D + 4 * t) = make_float4(a2[0] / B, a2[1] / B, a2[2] / B, a2[3] / B);
  }
}

// Levels 3..L, one CTA per slice: each level from the one below it in global
// memory (written by this CTA, or by the previous launch for level 2), with
// the same per-token arithmetic as pool_level_kernel.
__global__ void __launch_bounds__(256) pool_upper_kernel(float* __restrict__ pyr, Geo g) {
  const int bh = blockIdx.x;
  const int c4n = g.d / 4;
  for (int l = 3; l <= g.L; ++l) {
    const float* prev = pyr + g.pyr_off[l - 1] + (int64_t)bh * g.n[l - 1] * g.d;
    float* out = pyr + g.pyr_off[l] + (int64_t)bh * g.n[l] * g.d;
    const int64_t total = (int64_t)g.n[l] * c4n;
    for (int64_t e = threadIdx.x; e < total; e += blockDim.x) {
      const int64_t tok = e / c4n;
      const int c = (int)(e - tok * c4n) * 4;
      const float* src = prev + tok * g.B * g.d + c;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int r = 0; r < g.B; ++r) {
        const float4 w = *reinterpret_cast<const float4*>(src + (int64_t)r * g.d);
        acc[0] += w.x; acc[1] += w.y; acc[2] += w.z; acc[3] += w.w;
      }
      *reinterpret_cast<float4*>(out + tok * g.d + c) =
          make_float4(acc[0] / g.B, acc[1] / g.B, acc[2] / g.B, acc[3] / g.B);
    }
    __syncthreads();   // the level is complete before the next one reads it
  }
}

cudaError_t launch_pool(const Geo& g, const void* x, float* pyr, cudaStream_t s) {
  if (g.B == 16 && g.d == 64 && g.L >= 2) {
    const unsigned grid = (unsigned)((int64_t)g.BH * g.n[2]);
    if (g.bf16)
      pool_l12_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16*)x, pyr + g.pyr_off[1],
                                                            pyr + g.pyr_off[2]);
    else
      pool_l12_kernel<float><<<grid, 256, 0, s>>>((const float*)x, pyr + g.pyr_off[1], pyr + g.pyr_off[2]);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || g.L < 3) return e;
    pool_upper_kernel<<<g.BH, 256, 0, s>>>(pyr, g);
    note_launches(1);
    return cudaGetLastError();
  }
  for (int l = 1; l <= g.L; ++l) {
    int64_t total = (int64_t)g.BH * g.n[l] * (g.d / 4);
    float* out = pyr + g.pyr_off[l];
    if (l == 1) {
      if (g.bf16)
        pool_launch((const __nv_bfloat16*)x, out, g, total, s);
      else
        pool_launch((const float*)x, out, g, total, s);
    } else {
      pool_launch((const float*)(pyr + g.pyr_off[l - 1]), out, g, total, s);
    }
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace llsa
