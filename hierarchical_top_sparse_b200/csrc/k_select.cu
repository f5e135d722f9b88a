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
#include "ptx.cuh"

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

// ------------------------------------------------ child search, pipelined over parents
//
// The B sibling query tokens under one level-(l+1) token (a parent) share
// their candidates: the B children of each of the parent's picks.  A CTA
// walks parents in grid-stride order with two shared-memory stages: the
// candidate rows and the 16 query rows of parent i + 2 are copied in
// (16-byte asynchronous copies into padded rows) while the CTA scores parent
// i.  Every thread scores a 2 x 4 register tile (2 query rows of its warp x
// candidates lane + 32 j), each a sequential fp32 FMA chain over the 64
// channels; then the warp takes K_l rounds of a warp-wide maximum for each of
// its rows (two one-instruction reductions per round: the orderable score,
// then, among the lanes that hold it, the lower candidate position) and
// writes the picks in ascending order.
namespace selchild {
constexpr int THREADS = 256;
constexpr int NC = 128;        // candidates per parent, at most (K_{l+1} <= 8)
constexpr int QB = 16;         // sibling query tokens (B)
constexpr int LD = 68;         // padded row length (floats): conflict-free 16-byte reads
constexpr int STAGES = 2;
struct Stage {
  float k[NC * LD];            // candidate m = child m % B of pick m / B
  float q[QB * LD];            // the parent's 16 query rows
};
constexpr size_t kSmem = sizeof(Stage) * STAGES;
static_assert((NC + QB) * 16 % THREADS == 0, "every thread copies the same number of 16-byte pieces");
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__global__ void __launch_bounds__(selchild::THREADS) select_children_kernel(Geo g, int l,
                                                                            const float* __restrict__ pyrQ,
                                                                            const float* __restrict__ pyrK,
                                                                            int32_t* __restrict__ idx) {
  using namespace selchild;
  extern __shared__ __align__(16) unsigned char sm_raw[];
  Stage* st = reinterpret_cast<Stage*>(sm_raw);
  __shared__ int cids[STAGES][NC];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nl = g.n[l], np = g.n[l + 1];
  const int Kp = g.Kl[l + 1], Kl = g.Kl[l];
  const int ncand = Kp * QB;
  const int64_t nparents = (int64_t)g.BH * np;
  const int64_t stride = gridDim.x;

  // Stage sidx <- parent p (every thread copies its share); one copy group
  // per call, empty when p is past the end.  Candidate ids < 0: the pick lies
  // outside its level (-1 - the id the list implies), the candidate never wins.
  auto issue = [&](int64_t p, int sidx) {
    if (p < nparents) {
      const int bh = (int)(p / np), par = (int)(p - (int64_t)bh * np);
      const int32_t* plist = idx + g.idx_off[l + 1] + ((int64_t)bh * np + par) * Kp;
      const float* kbase = pyrK + g.pyr_off[l] + (int64_t)bh * nl * 64;
      const float* qbase = pyrQ + g.pyr_off[l] + ((int64_t)bh * nl + (int64_t)par * QB) * 64;
      // lane j of every warp holds pick j: one round of loads, then shuffles
      const int pl = lane < Kp ? plist[lane] : -1;
      if (tid < NC) {
        const int pc = __shfl_sync(0xffffffffu, pl, (tid / QB) & 31);
        cids[sidx][tid] = tid >= ncand ? -1
                          : (pc >= 0 && pc < np) ? pc * QB + tid % QB : -1 - (pc * QB + tid % QB);
      }
#pragma unroll 1
      for (int e = tid; e < (NC + QB) * 16; e += THREADS) {   // the same trip count in every thread
        const int r = e >> 4, c4 = (e & 15) * 4;
        const int pc = __shfl_sync(0xffffffffu, pl, (r / QB) & 31);
        if (r < NC) {
          if (r < ncand && pc >= 0 && pc < np)
            cp_async16(&st[sidx].k[r * LD + c4], kbase + ((int64_t)pc * QB + r % QB) * 64 + c4);
        } else {
          cp_async16(&st[sidx].q[(r - NC) * LD + c4], qbase + (r - NC) * 64 + c4);
        }
      }
    }
    cp_async_commit();
  };

  const int64_t first = blockIdx.x;
  issue(first, 0);
  issue(first + stride, 1);
  uint32_t it = 0;
  for (int64_t p = first; p < nparents; p += stride, ++it) {
    const int sidx = (int)(it & 1);
    cp_async_wait_one();   // this stage's copies (the next stage's may still fly)
    __syncthreads();
    const Stage& S = st[sidx];
    // scores: warp w takes query rows 2w, 2w+1, lane the candidates lane + 32 j
    float acc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int e = 0; e < 64; e += 4) {
      float4 qv[2], kv[4];
#pragma unroll
      for (int i = 0; i < 2; ++i) qv[i] = *reinterpret_cast<const float4*>(&S.q[(warp * 2 + i) * LD + e]);
#pragma unroll
      for (int j = 0; j < 4; ++j) kv[j] = *reinterpret_cast<const float4*>(&S.k[(lane + 32 * j) * LD + e]);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(qv[i].x, kv[j].x, acc[i][j]);
          acc[i][j] = fmaf(qv[i].y, kv[j].y, acc[i][j]);
          acc[i][j] = fmaf(qv[i].z, kv[j].z, acc[i][j]);
          acc[i][j] = fmaf(qv[i].w, kv[j].w, acc[i][j]);
        }
    }
    int cid[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) cid[j] = cids[sidx][lane + 32 * j];
    const int bh = (int)(p / np), par = (int)(p - (int64_t)bh * np);
    __syncthreads();   // every read of this stage is done: refill it
    issue(p + 2 * stride, sidx);

    // keys: hi = orderable score (0: no score), lo = 128 - candidate position
    // (0: no candidate or taken); the maximum (hi, lo) is the highest score,
    // then the lowest position, i.e. the lowest key id
    uint32_t hi[2][4], lo[2][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = lane + 32 * j;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (m >= ncand) {
          hi[i][j] = 0u;
          lo[i][j] = 0u;
        } else {
          hi[i][j] = cid[j] < 0 ? 0u : orderable(acc[i][j]);   // a pick outside its level: after every score
          lo[i][j] = 128u - (uint32_t)m;
        }
      }
    }
    unsigned taken[2] = {0u, 0u};
    for (int k = 0; k < Kl; ++k) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        uint32_t bh_ = hi[i][0], bl_ = lo[i][0];
#pragma unroll
        for (int j = 1; j < 4; ++j)
          if (hi[i][j] > bh_ || (hi[i][j] == bh_ && lo[i][j] > bl_)) {
            bh_ = hi[i][j];
            bl_ = lo[i][j];
          }
        const uint32_t H = __reduce_max_sync(0xffffffffu, bh_);
        const uint32_t Lw = __reduce_max_sync(0xffffffffu, bh_ == H ? bl_ : 0u);
        const int m = 128 - (int)Lw;
        const bool mine = (m & 31) == lane;
        const int jj = m >> 5;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (mine && j == jj) {
            hi[i][j] = 0u;
            lo[i][j] = 0u;
          }
        if (mine) taken[i] |= 1u << jj;
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int r = warp * 2 + i;
      int32_t* out = idx + g.idx_off[l] + ((int64_t)bh * nl + (int64_t)par * QB + r) * Kl;
      int written = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool t = (taken[i] >> j) & 1u;
        const unsigned bal = __ballot_sync(0xffffffffu, t);
        if (t) out[written + __popc(bal & ((1u << lane) - 1u))] = cid[j] >= 0 ? cid[j] : -1 - cid[j];
        written += __popc(bal);
      }
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");   // nothing in flight when the CTA leaves
}

cudaError_t launch_select_level(const Geo& g, int level, const float* pyrQ, const float* pyrK, int32_t* idx,
                                cudaStream_t s) {
  if (level < g.L && g.d == 64 && g.B == selchild::QB && g.Kl[level + 1] * g.B <= selchild::NC &&
      g.Kl[level] < g.Kl[level + 1] * g.B) {
    const int64_t parents = (int64_t)g.BH * g.n[level + 1];
    cudaError_t e = cudaFuncSetAttribute(select_children_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)selchild::kSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t resident = 2ll * sms;   // two CTAs of 77 KB per SM
    const unsigned grid = (unsigned)(parents < resident ? parents : resident);
    select_children_kernel<<<grid, selchild::THREADS, selchild::kSmem, s>>>(g, level, pyrQ, pyrK, idx);
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
