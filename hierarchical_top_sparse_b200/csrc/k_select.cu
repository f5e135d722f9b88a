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

// ------------------------------------------------ child search, one CTA per parent
//
// The B sibling query tokens under one level-(l+1) token share their
// candidates (the B children of each of the parent's picks), so one CTA
// loads those candidate rows once into shared memory and scores the whole
// B x (K_{l+1} B) tile: every thread a 4 x 4 register tile of scores, each a
// sequential fp32 FMA chain over d (the same rounding as the one-warp kernel
// above).  Then one warp per query token takes K_l rounds of a warp-wide max
// over 64-bit keys held in registers and writes the picks in ascending order.
namespace selchild {
constexpr int THREADS = 128;
constexpr int NC = 128;        // candidates per parent, at most
constexpr int QB = 16;         // sibling query tokens (B)
constexpr int LD = 68;         // padded row length (floats): conflict-free 16-byte reads
}

__global__ void __launch_bounds__(selchild::THREADS) select_children_kernel(Geo g, int l,
                                                                            const float* __restrict__ pyrQ,
                                                                            const float* __restrict__ pyrK,
                                                                            int32_t* __restrict__ idx) {
  using namespace selchild;
  __shared__ __align__(16) float ks[NC * LD];
  __shared__ __align__(16) float qs[QB * LD];
  __shared__ int cid[NC];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nl = g.n[l], np = g.n[l + 1];
  const int bh = blockIdx.x / np;
  const int par = blockIdx.x - bh * np;
  const int Kp = g.Kl[l + 1], Kl = g.Kl[l];
  const int ncand = Kp * QB;
  const int32_t* plist = idx + g.idx_off[l + 1] + ((int64_t)bh * np + par) * Kp;
  const float* kbase = pyrK + g.pyr_off[l] + (int64_t)bh * nl * 64;
  const float* qbase = pyrQ + g.pyr_off[l] + ((int64_t)bh * nl + (int64_t)par * QB) * 64;

  // Candidate m is child m % B of pick m / B.  Every thread resolves the ids of
  // the rows it copies itself (the parent list is a few cached words), so the
  // candidate rows and the query rows are fetched in one round.
  auto cand = [&](int m) -> int {
    if (m >= ncand) return -1;
    const int pc = plist[m / QB];
    return (pc >= 0 && pc < np) ? pc * QB + m % QB : -1 - (pc * QB + m % QB);   // < 0: parent corrupted
  };
  if (tid < NC) cid[tid] = cand(tid);
  for (int e = tid; e < QB * 16; e += THREADS) {
    const int r = e >> 4, c4 = (e & 15) * 4;
    *reinterpret_cast<float4*>(&qs[r * LD + c4]) = *reinterpret_cast<const float4*>(qbase + r * 64 + c4);
  }
  for (int e = tid; e < NC * 16; e += THREADS) {
    const int m = e >> 4, c4 = (e & 15) * 4;
    const int c = cand(m);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c >= 0) v = *reinterpret_cast<const float4*>(kbase + (int64_t)c * 64 + c4);
    *reinterpret_cast<float4*>(&ks[m * LD + c4]) = v;
  }
  __syncthreads();

  // scores: warp w takes query rows 4w..4w+3, lane the candidates lane + 32 j;
  // they stay in registers
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int e = 0; e < 64; e += 4) {
    float4 qv[4], kv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) qv[i] = *reinterpret_cast<const float4*>(&qs[(warp * 4 + i) * LD + e]);
#pragma unroll
    for (int j = 0; j < 4; ++j) kv[j] = *reinterpret_cast<const float4*>(&ks[(lane + 32 * j) * LD + e]);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[i][j] = fmaf(qv[i].x, kv[j].x, acc[i][j]);
        acc[i][j] = fmaf(qv[i].y, kv[j].y, acc[i][j]);
        acc[i][j] = fmaf(qv[i].z, kv[j].z, acc[i][j]);
        acc[i][j] = fmaf(qv[i].w, kv[j].w, acc[i][j]);
      }
  }

  // top-K_l of the warp's 4 rows, the 4 rows' rounds interleaved so that their
  // shuffle chains overlap: 64-bit keys (orderable score, then the lower
  // candidate position wins a tie)
  uint64_t key[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int m = lane + 32 * j;
    const int c = m < ncand ? cid[m] : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (m >= ncand)
        key[i][j] = 0;
      else if (c < 0)
        key[i][j] = 1ull << 32;          // parent corrupted: the candidate never wins
      else
        key[i][j] = ((uint64_t)orderable(acc[i][j]) << 32) | (uint64_t)(0xffffffffu - (uint32_t)m);
    }
  }
  unsigned taken[4] = {0u, 0u, 0u, 0u};
  for (int k = 0; k < Kl; ++k) {
    uint64_t best[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      best[i] = key[i][0];
#pragma unroll
      for (int j = 1; j < 4; ++j) best[i] = key[i][j] > best[i] ? key[i][j] : best[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t w = __shfl_xor_sync(0xffffffffu, best[i], o);
        best[i] = w > best[i] ? w : best[i];
      }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = (int)(0xffffffffu - (uint32_t)best[i]);
      const bool mine = (m & 31) == lane;
      const int jj = m >> 5;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (mine && j == jj) key[i][j] = 0;
      if (mine) taken[i] |= 1u << jj;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = warp * 4 + i;
    int32_t* out = idx + g.idx_off[l] + ((int64_t)bh * nl + (int64_t)par * QB + r) * Kl;
    int written = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool t = (taken[i] >> j) & 1u;
      const unsigned bal = __ballot_sync(0xffffffffu, t);
      if (t) {
        const int m = lane + 32 * j;
        const int c = cid[m];
        out[written + __popc(bal & ((1u << lane) - 1u))] = c >= 0 ? c : -1 - c;
      }
      written += __popc(bal);
    }
  }
}

cudaError_t launch_select_level(const Geo& g, int level, const float* pyrQ, const float* pyrK, int32_t* idx,
                                cudaStream_t s) {
  if (level < g.L && g.d == 64 && g.B == selchild::QB && g.Kl[level + 1] * g.B <= selchild::NC &&
      g.Kl[level] < g.Kl[level + 1] * g.B) {
    const int64_t parents = (int64_t)g.BH * g.n[level + 1];
    select_children_kernel<<<(unsigned)parents, selchild::THREADS, 0, s>>>(g, level, pyrQ, pyrK, idx);
    note_launches(1);
    return cudaGetLastError();
  }
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
