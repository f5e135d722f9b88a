// k_attn_fwd_mma.cu -- sparse attention forward on the tensor cores (bf16,
// d = 64, B = 16).
//
// Work unit: a group of 8 sibling query blocks (128 fine queries under one
// level-2 parent).  The 8 blocks pick their K_1 key blocks among the same
// candidates, so their picks overlap; the group loads the UNION of its picks
// once.  One persistent CTA per SM, each on a contiguous range of groups:
//   * a union warp sorts and deduplicates the group's picks, a group ahead;
//   * a TMA warp streams the union's K/V blocks (2 KB each) with TMA 2-D
//     tile loads (128-byte swizzle) through a ring of slots guarded by
//     mbarriers, one lane per slot;
//   * 16 consumer warps, two per query block, convert the group's pooled
//     keys of levels >= 2 (shared by all 128 queries) to bf16 once per
//     level-2 parent; each warp then takes every other one of its block's
//     picks (and half of the pooled keys), walks the union in order and
//     feeds them through warp-level MMA (m16n8k16, bf16 in, fp32 accumulate)
//     with the online softmax in registers: exactly K_1 * B fine keys plus
//     the pooled keys per query, no masked work.  The second warp of a block
//     hands its running max, sum and O (as bf16) to the first through shared
//     memory, which merges them and writes O and LSE.
// A pooled level-1 token is the mean of the 16 keys of the block it stands
// for, so its logit is the mean of that block's 16 fine logits and its value
// term spreads P_c / B onto the block's 16 values: level-1 enrichment costs no
// extra load and no extra MMA (hierarchical KV enrichment and KV reweighting,
// Trainable Log-linear Sparse Attention summary §四).
#include <math.h>

#include "llsa_internal.cuh"
#include "ptx.cuh"

namespace llsa {

namespace fwdmma {

constexpr int G = 8;             // query blocks per group = consumer warps
constexpr int SLOTS = 32;        // ring slots, each one K block and one V block
constexpr int NBUF = 3;          // groups in flight (query tiles, union lists)
constexpr int COARSE = 32;       // pooled keys of levels >= 2 per group, at most
constexpr int MAXPICK = 256;     // G * K_1, at most
constexpr int MAXWORDS = 2048;   // union bitmap: level-1 blocks per slice, at most 65536
constexpr int CW = 2;            // consumer warps per query block: each takes every other pick
constexpr int BATCH = 1;         // picked blocks per softmax batch
constexpr int TMA_WARP = CW * G;
constexpr int UNION_WARP = CW * G + 1;
constexpr int THREADS = (CW * G + 2) * 32;
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s: a wait this long means something broke

struct Smem {
  alignas(1024) unsigned char ring[SLOTS][4096];
  alignas(1024) unsigned char q[NBUF][G][2048];
  alignas(1024) unsigned char ck[COARSE * 128];
  alignas(1024) unsigned char cv[COARSE * 128];
  float cbias[COARSE];
  int crow_l[COARSE];
  int crow_tok[COARSE];
  int ulist[NBUF][MAXPICK];
  uint32_t pickpos[NBUF][MAXPICK];   // ring position of every pick, in pick order
  int ucnt[NBUF][MAXPICK];           // how many of the group's blocks picked union entry u
  unsigned bitmap[MAXWORDS];
  int ucount[NBUF];
  uint32_t issued[SLOTS];  // ring position whose copy was last issued into each slot
  alignas(8) uint64_t full[SLOTS];
  uint64_t empty[SLOTS];
  uint64_t qfull[NBUF];    // query tiles landed (TMA) and the union list written
  uint64_t qempty[NBUF];   // the group's consumers are done with the buffer
  uint64_t ufull[NBUF];    // the union list is written: union warp -> TMA warp
  uint64_t csync;          // consumer-wide barrier around the pooled-key tile
  // a query block's second consumer warp hands its partial state to the first:
  // O as bf16 pairs in the fragment layout ([word][lane]) and the row max and
  // sum of rows gq, gq + 8 (log2 domain)
  uint32_t part[G][16][32];
  float pstat[G][4][32];
  uint64_t mfull[G], mempty[G];
  int abort_flag;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA exceeds the 227 KB limit");

__device__ __forceinline__ void give_up(Smem& s, int* err, int code) {
  s.abort_flag = 1;
  if (err) atomicExch(err, code);
}

__device__ __forceinline__ bool aborted(Smem& s) { return *(volatile int*)&s.abort_flag != 0; }

// All G consumer warps meet on an mbarrier (a bounded wait, unlike bar.sync,
// so a consumer that gave up cannot hang the others).
__device__ __forceinline__ bool consumers_sync(Smem& s, uint32_t& phase) {
  ptx::mbar_arrive(&s.csync);
  const bool ok = ptx::mbar_wait_bounded(&s.csync, phase & 1, kWaitLimitNs);
  ++phase;
  return ok;
}

__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  return fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

struct RowState {
  float m[2];     // running max (log2 domain) of rows g and g+8
  float l[2];     // running partial sums (this lane's columns)
  float acc[8][4];
};

__device__ __forceinline__ void rescale(RowState& st, float mn0, float mn1) {
  const float a0 = ptx::ex2(st.m[0] - mn0), a1 = ptx::ex2(st.m[1] - mn1);
  st.m[0] = mn0;
  st.m[1] = mn1;
  st.l[0] *= a0;
  st.l[1] *= a1;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    st.acc[j][0] *= a0;
    st.acc[j][1] *= a0;
    st.acc[j][2] *= a1;
    st.acc[j][3] *= a1;
  }
}

// O += P (16 x 16 keys, bf16 A fragment) * V (16 keys x 64, swizzled tile at vbase)
__device__ __forceinline__ void pv_16(RowState& st, const uint32_t* pa, uint32_t vbase, int key0, int lane) {
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    // matrices: [keys 0-7, d 8j..], [keys 8-15, d 8j..], [keys 0-7, d 8j+8..], [keys 8-15, d 8j+8..]
    const int row = key0 + (lane & 7) + (((lane >> 3) & 1) << 3);
    const int col = (j + (lane >> 4)) * 8;
    uint32_t b0, b1, b2, b3;
    ptx::ldmatrix_x4_trans(vbase + ptx::sw128(row, col), b0, b1, b2, b3);
    ptx::mma_bf16(st.acc[j], pa, b0, b1);
    ptx::mma_bf16(st.acc[j + 1], pa, b2, b3);
  }
}

// S (16 x 16) = Q (A fragments, 4 k-steps) * K^T, keys key0..key0+15 of the tile at kbase
__device__ __forceinline__ void qk_16(float (*s)[4], const uint32_t (*qa)[4], uint32_t kbase, int key0, int lane) {
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[j][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    // matrices: [keys 0-7, d lo], [keys 0-7, d hi], [keys 8-15, d lo], [keys 8-15, d hi]
    const int row = key0 + (lane & 7) + ((lane >> 4) << 3);
    const int col = ks * 16 + (((lane >> 3) & 1) << 3);
    uint32_t b0, b1, b2, b3;
    ptx::ldmatrix_x4(kbase + ptx::sw128(row, col), b0, b1, b2, b3);
    ptx::mma_bf16(s[0], qa[ks], b0, b1);
    ptx::mma_bf16(s[1], qa[ks], b2, b3);
  }
}

// Ascending bitonic sort of 64 values held 2 per lane (element 2*lane + r).
__device__ __forceinline__ void warp_sort64(int& x0, int& x1, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 1) {
        const bool up = ((2 * lane) & k) == 0;
        const int lo = min(x0, x1), hi = max(x0, x1);
        x0 = up ? lo : hi;
        x1 = up ? hi : lo;
      } else {
        const int y0 = __shfl_xor_sync(0xffffffffu, x0, j >> 1);
        const int y1 = __shfl_xor_sync(0xffffffffu, x1, j >> 1);
        const int e0 = 2 * lane, e1 = 2 * lane + 1;
        const bool up0 = (e0 & k) == 0, low0 = (e0 & j) == 0;
        const bool up1 = (e1 & k) == 0, low1 = (e1 & j) == 0;
        x0 = (low0 == up0) ? min(x0, y0) : max(x0, y0);
        x1 = (low1 == up1) ? min(x1, y1) : max(x1, y1);
      }
    }
  }
}

// Softmax batch: up to BATCH picked fine blocks of one query block (16 rows).
// pslots packs the ring slots of the pending blocks, 5 bits each.
__device__ __forceinline__ void fine_batch(RowState& st, const uint32_t (*qa)[4], Smem& s, uint32_t pslots,
                                           int npend, int lane, int tq4, float sc2, float log2B, bool enrich1) {
  float z[BATCH][2][4];
  float zc[BATCH][2];
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < BATCH; ++i) {
    if (i < npend) {
      qk_16(z[i], qa, ptx::smem_u32(s.ring[(pslots >> (5 * i)) & 31]), 0, lane);
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) z[i][j][e] *= sc2;
        mx0 = fmaxf(mx0, fmaxf(z[i][j][0], z[i][j][1]));
        mx1 = fmaxf(mx1, fmaxf(z[i][j][2], z[i][j][3]));
        sum0 += z[i][j][0] + z[i][j][1];
        sum1 += z[i][j][2] + z[i][j][3];
      }
      if (enrich1) {
        // the pooled level-1 token of this block: mean of its 16 fine logits, weight B
        zc[i][0] = quad_sum(sum0) * (1.f / 16.f) + log2B;
        zc[i][1] = quad_sum(sum1) * (1.f / 16.f) + log2B;
        mx0 = fmaxf(mx0, zc[i][0]);
        mx1 = fmaxf(mx1, zc[i][1]);
      }
    }
  }
  mx0 = quad_max(mx0);
  mx1 = quad_max(mx1);
  const float mn0 = fmaxf(st.m[0], mx0), mn1 = fmaxf(st.m[1], mx1);
  rescale(st, mn0, mn1);
#pragma unroll
  for (int i = 0; i < BATCH; ++i) {
    if (i < npend) {
      float sh0 = 0.f, sh1 = 0.f;
      if (enrich1) {
        const float pc0 = ptx::ex2(zc[i][0] - mn0), pc1 = ptx::ex2(zc[i][1] - mn1);
        if (tq4 == 0) {
          st.l[0] += pc0;
          st.l[1] += pc1;
        }
        sh0 = pc0 * (1.f / 16.f);
        sh1 = pc1 * (1.f / 16.f);
      }
      float p[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        p[j][0] = ptx::ex2(z[i][j][0] - mn0);
        p[j][1] = ptx::ex2(z[i][j][1] - mn0);
        p[j][2] = ptx::ex2(z[i][j][2] - mn1);
        p[j][3] = ptx::ex2(z[i][j][3] - mn1);
        st.l[0] += p[j][0] + p[j][1];
        st.l[1] += p[j][2] + p[j][3];
      }
      uint32_t pa[4];
      pa[0] = ptx::pack_bf16(p[0][0] + sh0, p[0][1] + sh0);
      pa[1] = ptx::pack_bf16(p[0][2] + sh1, p[0][3] + sh1);
      pa[2] = ptx::pack_bf16(p[1][0] + sh0, p[1][1] + sh0);
      pa[3] = ptx::pack_bf16(p[1][2] + sh1, p[1][3] + sh1);
      pv_16(st, pa, ptx::smem_u32(s.ring[(pslots >> (5 * i)) & 31]) + 2048, 0, lane);
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1) attn_fwd_mma_kernel(
    const __grid_constant__ Geo g, const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, const float* __restrict__ pyrK, const float* __restrict__ pyrV,
    const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int* err,
    int groups_per_slice, int ngroups) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K1 = g.Kl[1];
  const float log2B = log2f((float)g.B);
  const float sc2 = g.scale * 1.4426950408889634f;   // logits in the log2 domain
  const bool enrich1 = g.emask & 1u;

  // pooled rows of levels >= 2: row r belongs to a fixed level for the whole launch
  int nc = 0;
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];

  if (threadIdx.x == 0) {
    for (int i = 0; i < SLOTS; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], G);
      s.issued[i] = 0xffffffffu;
    }
    for (int b = 0; b < NBUF; ++b) {
      ptx::mbar_init(&s.qfull[b], 2);     // the TMA bytes' arrival and the union list's arrival
      ptx::mbar_init(&s.qempty[b], CW * G);
      ptx::mbar_init(&s.ufull[b], 1);
    }
    for (int qb = 0; qb < G; ++qb) {
      ptx::mbar_init(&s.mfull[qb], 1);
      ptx::mbar_init(&s.mempty[qb], 1);
    }
    ptx::mbar_init(&s.csync, CW * G * 32);
    s.abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (threadIdx.x < COARSE) {
    const int r = threadIdx.x;
    int base = 0, lvl = 0;
    for (int l = 2; l <= g.L; ++l) {
      if (!((g.emask >> (l - 1)) & 1u)) continue;
      if (r >= base && r < base + g.Kl[l]) lvl = l;
      base += g.Kl[l];
    }
    s.crow_l[r] = lvl;
    s.cbias[r] = lvl ? (float)lvl * log2B : -INFINITY;
  }
  for (int w = threadIdx.x; w < MAXWORDS; w += blockDim.x) s.bitmap[w] = 0u;
  for (int e = threadIdx.x; e < COARSE * 32; e += blockDim.x) {     // zero both pooled tiles
    reinterpret_cast<uint32_t*>(s.ck)[e] = 0u;
    reinterpret_cast<uint32_t*>(s.cv)[e] = 0u;
  }
  __syncthreads();

  // Pairs of groups (the 16 blocks under one level-2 token) go to CTAs with a
  // grid stride: the CTAs in flight work on neighbouring groups of one
  // (batch, head) slice and share its K/V in L2.  Iteration `it` of this CTA
  // takes group group_of(it); the sequence is increasing.
  auto group_of = [&](int it) -> int {
    return 2 * ((int)blockIdx.x + (it >> 1) * (int)gridDim.x) + (it & 1);
  };

  if (warp == UNION_WARP) {
    // ----------------------------------------- union of the picks (a group ahead of the TMA warp)
    const int np = G * K1;
    const bool small = np <= 64;
    auto pick_ptr = [&](int gi) {
      const int bh = gi / groups_per_slice;
      const int a0 = (gi - bh * groups_per_slice) * G;
      return idx + g.idx_off[1] + ((int64_t)bh * g.n[1] + a0) * K1;   // the G lists are consecutive
    };
    int nx0 = 0x7fffffff, nx1 = 0x7fffffff;   // next group's picks (small case), prefetched
    if (small && group_of(0) < ngroups) {
      const int32_t* pk = pick_ptr(group_of(0));
      if (2 * lane < np) nx0 = pk[2 * lane];
      if (2 * lane + 1 < np) nx1 = pk[2 * lane + 1];
    }
    uint32_t ring_pos = 0;
    int it = 0;
    for (int gi = group_of(0); gi < ngroups; gi = group_of(++it)) {
      const int b = it % NBUF;
      const uint32_t use = (uint32_t)(it / NBUF);
      if (lane == 0 && !ptx::mbar_wait_bounded(&s.qempty[b], (use & 1) ^ 1, kWaitLimitNs)) give_up(s, err, 1);
      __syncwarp();
      if (aborted(s)) break;
      int nu = 0;
      int o0 = 0x7fffffff, o1 = 0x7fffffff;   // picks 2*lane, 2*lane+1 in pick order (small case)
      if (small) {
        int x0 = nx0, x1 = nx1;
        if (x0 < 0 || x0 >= g.n[1]) x0 = 0x7fffffff;
        if (x1 < 0 || x1 >= g.n[1]) x1 = 0x7fffffff;
        o0 = x0;
        o1 = x1;
        nx0 = nx1 = 0x7fffffff;
        if (group_of(it + 1) < ngroups) {     // prefetch the next group's picks
          const int32_t* pk = pick_ptr(group_of(it + 1));
          if (2 * lane < np) nx0 = pk[2 * lane];
          if (2 * lane + 1 < np) nx1 = pk[2 * lane + 1];
        }
        warp_sort64(x0, x1, lane);
        const int prev = __shfl_up_sync(0xffffffffu, x1, 1);
        const bool f0 = x0 != 0x7fffffff && (lane == 0 || x0 != prev);
        const bool f1 = x1 != 0x7fffffff && x1 != x0;
        const unsigned b0 = __ballot_sync(0xffffffffu, f0), b1 = __ballot_sync(0xffffffffu, f1);
        const unsigned lt = (1u << lane) - 1u;
        const int pos0 = __popc(b0 & lt) + __popc(b1 & lt);
        if (f0) s.ulist[b][pos0] = x0;
        if (f1) s.ulist[b][pos0 + (f0 ? 1 : 0)] = x1;
        nu = __popc(b0) + __popc(b1);
      } else {
        // larger K_1: a bitmap over the slice's level-1 blocks
        const int32_t* pk = pick_ptr(gi);
        int lo = 0x7fffffff, hi = -1;
        for (int e = lane; e < np; e += 32) {
          const int v = pk[e];
          if (v >= 0 && v < g.n[1]) {
            atomicOr(&s.bitmap[v >> 5], 1u << (v & 31));
            lo = min(lo, v >> 5);
            hi = max(hi, v >> 5);
          }
        }
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) {
          lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o2));
          hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o2));
        }
        __syncwarp();
        for (int w0 = lo; w0 <= hi; w0 += 32) {
          const int w = w0 + lane;
          unsigned bits = w <= hi ? s.bitmap[w] : 0u;
          if (w <= hi && bits) s.bitmap[w] = 0u;        // leave the bitmap clear for the next group
          const int c = __popc(bits);
          int incl = c;
#pragma unroll
          for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o2);
            if (lane >= o2) incl += y;
          }
          int pos = nu + incl - c;
          while (bits) {
            const int bit = __ffs(bits) - 1;
            bits &= bits - 1;
            s.ulist[b][pos++] = w * 32 + bit;
          }
          nu += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
      if (lane == 0) s.ucount[b] = nu;
      for (int u = lane; u < nu; u += 32) s.ucnt[b][u] = 0;
      __syncwarp();
      // ring position of every pick (binary search in the sorted union) and the
      // number of the group's blocks that use each union entry
      {
        const int32_t* pk = pick_ptr(gi);
        for (int e = (small ? 2 * lane : lane); e < np; e += (small ? 1 : 32)) {
          if (small && e > 2 * lane + 1) break;
          int v;
          if (small)
            v = (e == 2 * lane) ? o0 : o1;
          else
            v = pk[e];
          int lo2 = 0, hi2 = nu - 1, r = -1;
          while (lo2 <= hi2) {
            const int mid = (lo2 + hi2) >> 1;
            const int w = s.ulist[b][mid];
            if (w == v) { r = mid; break; }
            if (w < v) lo2 = mid + 1; else hi2 = mid - 1;
          }
          s.pickpos[b][e] = r >= 0 ? ring_pos + (uint32_t)r : 0xffffffffu;
          if (r >= 0) atomicAdd(&s.ucnt[b][r], 1);
        }
      }
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&s.qfull[b]);     // union list and pick positions visible to the consumers
        ptx::mbar_arrive(&s.ufull[b]);     // and to the TMA warp
      }
      ring_pos += (uint32_t)nu;
      __syncwarp();
    }
    return;
  }

  if (warp == TMA_WARP) {
    // ----------------------------------------- query tiles and the union's K/V blocks, TMA
    if (lane == 0) {
      ptx::prefetch_tmap(&tq);
      ptx::prefetch_tmap(&tk);
      ptx::prefetch_tmap(&tv);
    }
    uint32_t ring_pos = 0;
    int it = 0;
    for (int gi = group_of(0); gi < ngroups; gi = group_of(++it)) {
      const int b = it % NBUF;
      const uint32_t use = (uint32_t)(it / NBUF);
      const int bh = gi / groups_per_slice;
      const int a0 = (gi - bh * groups_per_slice) * G;
      if (lane == 0 && !ptx::mbar_wait_bounded(&s.qempty[b], (use & 1) ^ 1, kWaitLimitNs)) give_up(s, err, 1);
      __syncwarp();
      if (aborted(s)) break;
      if (lane == 0) ptx::mbar_arrive_expect_tx(&s.qfull[b], G * 2048);
      __syncwarp();
      if (lane < G) ptx::tma_load_2d(s.q[b][lane], &tq, 0, bh * g.N + (a0 + lane) * 16, &s.qfull[b]);
      if (lane == 0 && !ptx::mbar_wait_bounded(&s.ufull[b], use & 1, kWaitLimitNs)) give_up(s, err, 1);
      __syncwarp();
      if (aborted(s)) break;
      const int nu = s.ucount[b];
      // one lane per ring position
      bool ok = true;
      for (int u0 = 0; u0 < nu; u0 += 32) {
        const int u = u0 + lane;
        if (u < nu) {
          const uint32_t pos = ring_pos + u;
          const int slot = pos % SLOTS;
          if (!ptx::mbar_wait_bounded(&s.empty[slot], ((pos / SLOTS) & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
          } else {
            const int row = bh * g.N + s.ulist[b][u] * 16;
            ptx::mbar_arrive_expect_tx(&s.full[slot], 4096);
            ptx::tma_load_2d(s.ring[slot], &tk, 0, row, &s.full[slot]);
            ptx::tma_load_2d(s.ring[slot] + 2048, &tv, 0, row, &s.full[slot]);
            ptx::st_release_u32(&s.issued[slot], pos);
            // the blocks that did not pick this entry release the slot right away
            const int others = G - s.ucnt[b][u];
            if (others > 0) ptx::mbar_arrive_count(&s.empty[slot], (uint32_t)others);
          }
        }
        if (__any_sync(0xffffffffu, !ok)) break;
      }
      if (!ok) give_up(s, err, 2);
      ring_pos += nu;
      __syncwarp();
      if (aborted(s)) break;
    }
    // do not leave while copies this CTA issued may still be landing
    if (aborted(s)) {
      const uint32_t lo2 = ring_pos > SLOTS ? ring_pos - SLOTS : 0;
      for (uint32_t p = lo2 + lane; p < ring_pos; p += 32)
        ptx::mbar_wait_bounded(&s.full[p % SLOTS], (p / SLOTS) & 1, kWaitLimitNs);
      if (lane == 0)
        for (int j = it > NBUF - 1 ? it - NBUF + 1 : 0; j <= it && group_of(j) < ngroups; ++j)
          ptx::mbar_wait_bounded(&s.qfull[j % NBUF], (j / NBUF) & 1, kWaitLimitNs);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  // warp w takes query block w % G; half w / G of its picks (every other one)
  // and of its pooled keys, the second half handing its state to the first
  const int gq = lane >> 2, tq4 = lane & 3;
  const int qb = warp % G, half = warp / G;
  uint32_t cphase = 0;
  int64_t last_parent = -1;
  int it = 0;
  for (int gi = group_of(0); gi < ngroups; gi = group_of(++it)) {
    const int b = it % NBUF;
    const uint32_t use = (uint32_t)(it / NBUF);
    const int bh = gi / groups_per_slice;
    const int a0 = (gi - bh * groups_per_slice) * G;
    const int a = a0 + qb;

    // pooled keys of levels >= 2, once per level-2 parent (all 8 consumers)
    const int64_t parent = (int64_t)bh * g.n[1] + a0 / g.B;
    if (nc > 0 && parent != last_parent) {
      if (!consumers_sync(s, cphase)) {    // everyone is done with the previous tile
        give_up(s, err, 6);
        break;
      }
      if (threadIdx.x < nc) {
        const int l = s.crow_l[threadIdx.x];
        int r = threadIdx.x;
        for (int l2 = 2; l2 < l; ++l2)
          if ((g.emask >> (l2 - 1)) & 1u) r -= g.Kl[l2];
        const int64_t grp = a0 / g.Bl[l - 1];
        const int tok = idx[g.idx_off[l] + ((int64_t)bh * g.n[l] + grp) * g.Kl[l] + r];
        s.crow_tok[threadIdx.x] = (tok >= 0 && tok < g.n[l]) ? tok : -1;
      }
      if (!consumers_sync(s, cphase)) {
        give_up(s, err, 6);
        break;
      }
      for (int item = threadIdx.x; item < nc * 16; item += CW * G * 32) {
        const int row = item >> 4, chunk = item & 15;
        const int l = s.crow_l[row], tok = s.crow_tok[row];
        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
        if (tok >= 0) {
          const int64_t off = g.pyr_off[l] + ((int64_t)bh * g.n[l] + tok) * 64 + chunk * 4;
          kv = *reinterpret_cast<const float4*>(pyrK + off);
          vv = *reinterpret_cast<const float4*>(pyrV + off);
        }
        const uint32_t o2 = ptx::sw128(row, chunk * 4);
        *reinterpret_cast<uint2*>(s.ck + o2) =
            make_uint2(ptx::pack_bf16(kv.x, kv.y), ptx::pack_bf16(kv.z, kv.w));
        *reinterpret_cast<uint2*>(s.cv + o2) =
            make_uint2(ptx::pack_bf16(vv.x, vv.y), ptx::pack_bf16(vv.z, vv.w));
      }
      if (!consumers_sync(s, cphase)) {
        give_up(s, err, 6);
        break;
      }
      last_parent = parent;
    }

    if (!ptx::mbar_wait_bounded(&s.qfull[b], use & 1, kWaitLimitNs)) {
      give_up(s, err, 3);
      break;
    }
    // ring positions of this block's picks, lane j holding pick j (K_1 <= 32), ascending
    const uint32_t my_pos = lane < K1 ? s.pickpos[b][qb * K1 + lane] : 0xffffffffu;

    uint32_t qa[4][4];
    const uint32_t qbase = ptx::smem_u32(s.q[b][qb]);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const int row = lane & 15;
      const int col = ks * 16 + ((lane >> 4) << 3);
      ptx::ldmatrix_x4(qbase + ptx::sw128(row, col), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
    }
    RowState st;
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.acc[j][e] = 0.f;

    // pooled keys of levels >= 2, 16 at a time
    const uint32_t ckb = ptx::smem_u32(s.ck), cvb = ptx::smem_u32(s.cv);
    for (int k0 = 16 * half; k0 < nc; k0 += 16 * CW) {
      float sc[2][4];
      qk_16(sc, qa, ckb, k0, lane);
      float z[2][4];
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c0 = k0 + j * 8 + 2 * tq4;
        const float bb0 = s.cbias[c0], bb1 = s.cbias[c0 + 1];
        z[j][0] = fmaf(sc[j][0], sc2, bb0);
        z[j][1] = fmaf(sc[j][1], sc2, bb1);
        z[j][2] = fmaf(sc[j][2], sc2, bb0);
        z[j][3] = fmaf(sc[j][3], sc2, bb1);
        mx0 = fmaxf(mx0, fmaxf(z[j][0], z[j][1]));
        mx1 = fmaxf(mx1, fmaxf(z[j][2], z[j][3]));
      }
      mx0 = quad_max(mx0);
      mx1 = quad_max(mx1);
      const float mn0 = fmaxf(st.m[0], mx0), mn1 = fmaxf(st.m[1], mx1);
      rescale(st, mn0, mn1);
      uint32_t pa[4];
      float p[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        p[j][0] = ptx::ex2(z[j][0] - mn0);
        p[j][1] = ptx::ex2(z[j][1] - mn0);
        p[j][2] = ptx::ex2(z[j][2] - mn1);
        p[j][3] = ptx::ex2(z[j][3] - mn1);
        st.l[0] += p[j][0] + p[j][1];
        st.l[1] += p[j][2] + p[j][3];
      }
      pa[0] = ptx::pack_bf16(p[0][0], p[0][1]);
      pa[1] = ptx::pack_bf16(p[0][2], p[0][3]);
      pa[2] = ptx::pack_bf16(p[1][0], p[1][1]);
      pa[3] = ptx::pack_bf16(p[1][2], p[1][3]);
      pv_16(st, pa, cvb, k0, lane);
    }

    // the picked blocks, in ring order, in batches of up to BATCH
    uint32_t pslots = 0;      // ring slots of the pending blocks, 5 bits each
    int npend = 0;
    uint32_t first_pend = 0;
    bool ok = true;
    for (int j = half; j < K1; j += CW) {
      const uint32_t pos = __shfl_sync(0xffffffffu, my_pos, j);
      if (pos == 0xffffffffu) continue;           // a pick outside its level: absent key
      // a held slot returns to the ring before a later pick needs the same slot
      if (npend > 0 && pos >= first_pend + SLOTS) {
        fine_batch(st, qa, s, pslots, npend, lane, tq4, sc2, log2B, enrich1);
        __syncwarp();
        if (lane == 0)
          for (int i = 0; i < npend; ++i) ptx::mbar_arrive(&s.empty[(pslots >> (5 * i)) & 31]);
        npend = 0;
      }
      const int slot = pos % SLOTS;
      // A block skips the positions it did not pick, so the slot's barrier may
      // still be a whole phase behind, where a parity wait cannot tell phase u
      // from phase u - 2.  Once the producer has issued this position, every
      // earlier use of the slot has landed and been released, and the parity
      // wait below is exact.
      if (!ptx::wait_u32_equal(&s.issued[slot], pos, kWaitLimitNs) ||
          !ptx::mbar_wait_bounded(&s.full[slot], (pos / SLOTS) & 1, kWaitLimitNs)) {
        ok = false;
        break;
      }
      if (npend == 0) first_pend = pos;
      pslots = (npend == 0 ? 0u : pslots) | ((uint32_t)slot << (5 * npend));
      ++npend;
      if (npend == BATCH) {
        fine_batch(st, qa, s, pslots, npend, lane, tq4, sc2, log2B, enrich1);
        __syncwarp();
        if (lane == 0)
          for (int i = 0; i < npend; ++i) ptx::mbar_arrive(&s.empty[(pslots >> (5 * i)) & 31]);
        npend = 0;
      }
    }
    if (!ok) {
      give_up(s, err, 4);
      break;
    }
    if (npend > 0) {
      fine_batch(st, qa, s, pslots, npend, lane, tq4, sc2, log2B, enrich1);
      __syncwarp();
      if (lane == 0)
        for (int i = 0; i < npend; ++i) ptx::mbar_arrive(&s.empty[(pslots >> (5 * i)) & 31]);
      npend = 0;
    }
    if (aborted(s)) break;

    // epilogue: the second warp of the block hands over (m, l, O); the first
    // merges, O = acc / l, LSE = ln(sum) + max
    float l0 = quad_sum(st.l[0]), l1 = quad_sum(st.l[1]);
    const uint32_t mph = (uint32_t)(it & 1);
    if (half == 1) {
      if (!ptx::mbar_wait_bounded(&s.mempty[qb], mph ^ 1, kWaitLimitNs)) {
        give_up(s, err, 7);
        break;
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        s.part[qb][2 * jj][lane] = ptx::pack_bf16(st.acc[jj][0], st.acc[jj][1]);
        s.part[qb][2 * jj + 1][lane] = ptx::pack_bf16(st.acc[jj][2], st.acc[jj][3]);
      }
      s.pstat[qb][0][lane] = st.m[0];
      s.pstat[qb][1][lane] = st.m[1];
      s.pstat[qb][2][lane] = l0;
      s.pstat[qb][3][lane] = l1;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.mfull[qb]);
    } else {
      if (!ptx::mbar_wait_bounded(&s.mfull[qb], mph, kWaitLimitNs)) {
        give_up(s, err, 7);
        break;
      }
      const float m0b = s.pstat[qb][0][lane], m1b = s.pstat[qb][1][lane];
      const float mn0 = fmaxf(st.m[0], m0b), mn1 = fmaxf(st.m[1], m1b);
      const float a0 = ptx::ex2(st.m[0] - mn0), a1 = ptx::ex2(st.m[1] - mn1);
      const float b0 = ptx::ex2(m0b - mn0), b1 = ptx::ex2(m1b - mn1);
      l0 = l0 * a0 + s.pstat[qb][2][lane] * b0;
      l1 = l1 * a1 + s.pstat[qb][3][lane] * b1;
      const float inv0 = 1.f / l0, inv1 = 1.f / l1;
      const int64_t row0 = (int64_t)bh * g.N + (int64_t)a * 16 + gq;
      __nv_bfloat16* o0 = o + row0 * 64;
      __nv_bfloat16* o1 = o + (row0 + 8) * 64;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const uint32_t w0 = s.part[qb][2 * jj][lane], w1 = s.part[qb][2 * jj + 1][lane];
        const float2 p0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w0));
        const float2 p1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w1));
        const int c = jj * 8 + 2 * tq4;
        *reinterpret_cast<uint32_t*>(o0 + c) =
            ptx::pack_bf16((st.acc[jj][0] * a0 + p0.x * b0) * inv0, (st.acc[jj][1] * a0 + p0.y * b0) * inv0);
        *reinterpret_cast<uint32_t*>(o1 + c) =
            ptx::pack_bf16((st.acc[jj][2] * a1 + p1.x * b1) * inv1, (st.acc[jj][3] * a1 + p1.y * b1) * inv1);
      }
      if (tq4 == 0) {
        lse[row0] = (mn0 + log2f(l0)) * 0.6931471805599453f;
        lse[row0 + 8] = (mn1 + log2f(l1)) * 0.6931471805599453f;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.mempty[qb]);
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&s.qempty[b]);
  }
}

}  // namespace fwdmma

bool attn_fwd_mma_supported(const Geo& g) {
  if (!g.bf16 || g.d != 64 || g.B != 16) return false;
  if (g.n[1] > fwdmma::MAXWORDS * 32) return false;
  if (g.Kl[1] < 1 || g.Kl[1] > 32 || g.Kl[1] * fwdmma::G > fwdmma::MAXPICK) return false;
  if (g.n[1] % fwdmma::G) return false;
  int nc = 0;
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];
  if (nc > fwdmma::COARSE) return false;
  if ((int64_t)g.BH * g.N >= (1ll << 31)) return false;
  return true;
}

cudaError_t launch_attn_fwd_mma(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                                const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  cudaError_t e = make_token_map(&tq, q, (int64_t)g.BH * g.N);
  if (e == cudaSuccess) e = make_token_map(&tk, k, (int64_t)g.BH * g.N);
  if (e == cudaSuccess) e = make_token_map(&tv, v, (int64_t)g.BH * g.N);
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(fwdmma::Smem) + 1024;
  e = cudaFuncSetAttribute(fwdmma::attn_fwd_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int gps = g.n[1] / fwdmma::G;
  const int ngroups = g.BH * gps;
  const int npairs = (ngroups + 1) / 2;
  const int grid = npairs < sms ? npairs : sms;
  fwdmma::attn_fwd_mma_kernel<<<grid, fwdmma::THREADS, smem, s>>>(g, tq, tk, tv, pyrK, pyrV, idx,
                                                                  (__nv_bfloat16*)o, lse, device_error_word(), gps,
                                                                  ngroups);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace llsa
