// k_select.cu -- coarse-to-fine top-K block selection, one level per launch.
//
// Coarsest level: each level-L query token scores all n_L level-L keys.
// Finer level l: query token a scores only the B children of each pick of its
// parent floor(a/B) at level l+1 (hierarchical top-K, Trainable Log-linear
// Sparse Attention summary §三).  One warp per query token: the candidate
// scores go to shared memory as 64-bit keys (order-preserving score bits in the
// high word, inverted candidate position in the low word), so one warp-wide
// max gives "highest score, then lowest key id"; K_l rounds of that max pick
// the list, and a ballot pass writes it out in ascending key order (candidate
// ids grow with the candidate position because parent lists are ascending).
#include "llsa_internal.cuh"

namespace llsa {

__device__ __forceinline__ uint32_t orderable(float s) {
  uint32_t u = __float_as_uint(s);
  if (s != s) return 1u;                             // NaN ranks below every number
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    uint64_t w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

__global__ void select_level_kernel(Geo g, int l, const float* __restrict__ pyrQ, const float* __restrict__ pyrK,
                                    int32_t* __restrict__ idx, int warps, int cand_stride) {
  extern __shared__ uint64_t skey[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nl = g.n[l];
  const int64_t task = (int64_t)blockIdx.x * warps + warp;
  if (task >= (int64_t)g.BH * nl) return;
  const int bh = (int)(task / nl);
  const int a = (int)(task - (int64_t)bh * nl);
  const int d = g.d;
  const float* qrow = pyrQ + g.pyr_off[l] + ((int64_t)bh * nl + a) * d;
  const float* kbase = pyrK + g.pyr_off[l] + (int64_t)bh * nl * d;
  const int Kl = g.Kl[l];
  int ncand;
  const int32_t* par = nullptr;
  if (l == g.L) {
    ncand = nl;
  } else {
    const int Kp = g.Kl[l + 1];
    ncand = Kp * g.B;
    par = idx + g.idx_off[l + 1] + ((int64_t)bh * g.n[l + 1] + a / g.B) * Kp;
  }
  int32_t* out = idx + g.idx_off[l] + ((int64_t)bh * nl + a) * Kl;
  auto cand_id = [&](int m) -> int { return par ? par[m / g.B] * g.B + m % g.B : m; };
  const int parent_n = par ? g.n[l + 1] : 0;

  if (Kl >= ncand) {                       // fewer candidates than K: keep them all
    for (int m = lane; m < ncand; m += 32) out[m] = cand_id(m);
    return;
  }
  uint64_t* key = skey + (size_t)warp * cand_stride;
  for (int m = lane; m < ncand; m += 32) {
    if (par) {
      const int pc = par[m / g.B];
      if (pc < 0 || pc >= parent_n) {       // parent list corrupted: the candidate never wins
        key[m] = 1ull << 32;
        continue;
      }
    }
    const float* krow = kbase + (int64_t)cand_id(m) * d;
    float s = 0.f;
    for (int e = 0; e < d; e += 4) {
      float4 qv = *reinterpret_cast<const float4*>(qrow + e);
      float4 kv = *reinterpret_cast<const float4*>(krow + e);
      s = fmaf(qv.x, kv.x, s);
      s = fmaf(qv.y, kv.y, s);
      s = fmaf(qv.z, kv.z, s);
      s = fmaf(qv.w, kv.w, s);
    }
    key[m] = ((uint64_t)orderable(s) << 32) | (uint64_t)(0xffffffffu - (uint32_t)m);
  }
  __syncwarp();
  for (int r = 0; r < Kl; ++r) {
    uint64_t best = 0;
    for (int m = lane; m < ncand; m += 32) best = key[m] > best ? key[m] : best;
    best = warp_max_u64(best);
    const int m = (int)(0xffffffffu - (uint32_t)best);
    __syncwarp();
    if (lane == 0) key[m] = 0;             // taken
    __syncwarp();
  }
  int written = 0;
  for (int base = 0; base < ncand; base += 32) {
    const int m = base + lane;
    const bool taken = m < ncand && key[m] == 0;
    const unsigned bal = __ballot_sync(0xffffffffu, taken);
    if (taken) out[written + __popc(bal & ((1u << lane) - 1u))] = cand_id(m);
    written += __popc(bal);
  }
}

cudaError_t launch_select_level(const Geo& g, int level, const float* pyrQ, const float* pyrK, int32_t* idx,
                                cudaStream_t s) {
  const int nl = g.n[level];
  const int ncand = level == g.L ? nl : g.Kl[level + 1] * g.B;
  int warps = 8;
  size_t per_warp = (size_t)ncand * sizeof(uint64_t);
  const size_t budget = 192 * 1024;
  while (warps > 1 && per_warp * warps > budget) warps >>= 1;
  size_t smem = g.Kl[level] >= ncand ? 0 : per_warp * warps;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_level_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int64_t tasks = (int64_t)g.BH * nl;
  int grid = (int)((tasks + warps - 1) / warps);
  select_level_kernel<<<grid, warps * 32, smem, s>>>(g, level, pyrQ, pyrK, idx, warps, ncand);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace llsa
