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

static int grid_for(int64_t work, int threads) {
  int64_t blocks = (work + threads - 1) / threads;
  int64_t cap = 148ll * 16;
  return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

cudaError_t launch_reorder(const Geo& g, const void* in, void* out, int to_hier, cudaStream_t s) {
  int vec = g.d * (g.bf16 ? 2 : 4) / 16;
  int64_t total = (int64_t)g.BH * g.N * vec;
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

cudaError_t launch_pool(const Geo& g, const void* x, float* pyr, cudaStream_t s) {
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
