// k_attn_fwd_tc.cu -- sparse attention forward on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory), bf16, d = 64, B = 16.
//
// Follows the enrichment and reweighting of the Trainable Log-linear Sparse
// Attention summary (§四: the fine top-K key blocks plus the pooled tokens
// each enriched level selected, weight B^l) and the sparse-index forward of
// the popular write-up of arXiv:2512.16615 (§四: keys are gathered by index,
// no dense mask is built).
//
// Work unit: a level-2 token, two groups of 8 sibling query blocks (128
// queries each).  The key blocks that any block of a group picked (the union
// of the 8 sorted pick lists, each entry with an 8-bit mask of the query
// blocks that picked it) are taken 8 at a time: a chunk of 128 keys whose K
// and V tiles TMA stacks into 128-row, 128-byte-swizzled operands.  Per chunk:
//   S = Q_G K_c^T                     (M = 128 queries, N = 128 keys, K = 64)
//   one thread per (query row, pair of key blocks) reads its S values from
//   TMEM, takes the blocks its query block picked, adds each block's pooled
//   level-1 token (its logit is the mean of the block's 16 logits plus ln B,
//   its value the mean of the block's values, so it adds P_c / B to each of
//   the block's 16 weights) and writes P as bf16 pairs back to TMEM;
//   O += P V_c                        (M = 128, N = 64, K = 128 keys; A = P from TMEM)
// O is accumulated in TMEM over the group.  The pooled keys of levels >= 2 are
// the same for all 256 queries of the token: each group starts with one chunk
// against them (N = 32, logit bias l ln B).
//
// O += P V is issued one key block (16 keys, one K step) at a time and is not
// masked: the softmax threads write zero weights for the blocks their rows
// did not pick.  (tcgen05's per-lane output mask would skip those rows
// instead, but a masked MMA issues about three times slower than a plain
// one.)  The epilogue clears each O buffer after reading it.
//
// Online softmax with a lazy maximum: a row keeps its running maximum m and
// rescales O (in TMEM) only when a new logit exceeds m by more than 2^8, so
// the weights stay below 256 and O is rarely touched.
//
// Warp roles, one CTA per SM (25 warps):
//   * warp 23, union: forms each group's union of picks -- with at most 64
//     picks (K_1 <= 8, prefetched into registers a group ahead) by a
//     warp-wide bitonic sort of (block, query block) keys, otherwise by
//     merging the 8 sorted lists -- and writes every entry (a chunk of up to
//     8 key blocks, the pooled-key chunk, a group's end) straight into the
//     entry ring, with the TMA boxes of each chunk worked out: one box per
//     run of up to 4 consecutive key blocks; it also builds each token's tile
//     of pooled keys of levels >= 2 (bf16 rows in the swizzled operand
//     layout, logit bias per row);
//   * warps 20, 21, producers, on alternate entries: the chunk's K and V into
//     one of NSLOT slots, and the next group's Q (one 128-row box) into one of
//     three slots as the current group starts.  Issuing a TMA copy costs about
//     a hundred cycles whatever its size, so the boxes follow runs and two
//     warps issue in parallel;
//   * warps 22 and 24, MMA: converged warps whose elected lanes issue every
//     S (warp 22) and every O update (warp 24), so that the S of the next
//     entries never queues behind the issue of an O update;
//   * warps 0-15, softmax: one query row per thread; the four warps of a TMEM
//     subpartition take two key blocks of a chunk each (pooled keys: 16 each
//     in the first two), find their part of the row maximum and exchange it
//     through shared memory, so that all four take the same decision on the
//     running maximum and P is scaled alike across the row;
//   * warps 16-19, epilogue: O = acc / l and LSE out of the group's TMEM buffer
//     (two buffers: a group's epilogue overlaps the next group).
// Every hand-off is an mbarrier, every wait is bounded; on a timeout the
// kernel sets the device error word and stops.
#include <math.h>
#include <stddef.h>

#include "llsa_internal.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {
namespace fwdtc {

constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kHeadroom = 8.f;    // log2 of the largest weight before O is rescaled
constexpr int QG = 8;               // query blocks per group (128 queries)
constexpr int CK = 8;               // key blocks per chunk (128 keys)
constexpr int NSLOT = 4;            // K / V chunk slots
constexpr int NQ = 3;               // Q slots: the next group's Q lands while the last two finish
constexpr int NMETA = 16;           // entries in flight between the union warp and the others
constexpr int COARSE = 32;          // pooled keys of levels >= 2 per token, at most
constexpr int STAGE = 512;          // pick-list words a group stages in shared memory
constexpr int SOFT_WARPS = 16;      // four per TMEM subpartition, each on two of a chunk's key blocks
constexpr int PARTS = SOFT_WARPS / 4;
constexpr int NPROD = 2;            // producer warps, on alternate entries
constexpr int EPI0 = 16, PRODUCER0 = 20, MMA_WARP = 22, UNION_WARP = 23, PV_WARP = 24;
constexpr int THREADS = 25 * 32;
constexpr uint32_t TMEM_COLS = 512;
// S of entry buffer b at 128 b, its P (bf16 pairs) at 256 + 64 b, O of group buffer o at 384 + 64 o
constexpr uint32_t COL_S = 0, COL_P = 256, COL_O = 384;
constexpr unsigned kNone = 0x7fffffffu;
enum : int { kEnd = 0, kChunk = 1, kCoarse = 2, kGroupEnd = 3 };
constexpr int kFirst = 1;           // first entry of a group
// an entry is read by the two MMA warps, every softmax warp and the producer that loads it
constexpr int META_ARRIVALS = 2 + SOFT_WARPS + 1;

struct ChunkSlot {
  alignas(1024) unsigned char k[CK * 2048];    // [128 keys][64] bf16, 128-byte swizzle
  alignas(1024) unsigned char v[CK * 2048];
};

struct QSlot {
  alignas(1024) unsigned char q[QG * 2048];    // [128 queries][64] bf16, 128-byte swizzle
};

struct alignas(1024) CoarseSlot {
  unsigned char k[COARSE * 128];               // [32 pooled keys][64] bf16, 128-byte swizzle
  unsigned char v[COARSE * 128];
  float bias[COARSE];                          // logit bias (log2 domain); -inf: no key
};

struct Meta {                                  // union warp -> producers, MMA and softmax warps
  int kind, nq, flags;
  int gc, tk, kc;                              // the CTA's group, token and chunk counts
  int qrow;                                    // first entry of a group: the next group's first Q row, or -1
  int msk[CK];                                 // bit j: query block j of the group picked key block
  int row[CK];                                 // first K / V row of each key block
  int box[CK];                                 // key blocks in the TMA box starting at this block (0: none)
};

struct Smem {
  ChunkSlot slot[NSLOT];
  QSlot qs[NQ];
  CoarseSlot crs[2];
  Meta meta[NMETA];
  int stage[STAGE];
  float stat_m[2][128], stat_l[2][PARTS][128]; // a group's row maxima and (per part) sums: softmax -> epilogue
  float xmax[2][PARTS][128];                   // the parts' row maxima of an entry (by entry parity)
  alignas(8) uint64_t kfull[NSLOT], kempty[NSLOT];   // K / V slots: producer -> MMA, MMA -> producer
  uint64_t mfull[NMETA], mempty[NMETA];        // entries: union warp -> the rest, back
  uint64_t qfull[NQ], qempty[NQ];              // Q slots: producer -> MMA, MMA -> producer
  uint64_t cfull[2], cempty[2];                // pooled-key tiles: union warp -> MMA / softmax, back
  uint64_t s_full[2], s_empty[2];              // S buffers: MMA -> softmax, softmax warps -> MMA
  uint64_t p_full[2], p_empty[2];              // P buffers: softmax warps -> MMA, MMA -> softmax
  uint64_t o_full[2], o_empty[2];              // O buffers: MMA -> epilogue, epilogue (4 warps) -> MMA / softmax
  uint64_t st_full[2];                         // row statistics: softmax warps -> epilogue
  uint64_t xbar[4];                            // the softmax warps of a subpartition exchange their maxima
  uint64_t drain[2];
  uint32_t tmem_base;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA exceeds the 227 KB limit");
static_assert(sizeof(ChunkSlot) % 1024 == 0 && sizeof(QSlot) % 1024 == 0 && sizeof(CoarseSlot) % 1024 == 0,
              "operands are addressed with fixed strides");

__device__ __forceinline__ void report(int* err, int code) {
  if (err) atomicExch(err, code);
}

// Ascending bitonic sort of 64 keys held two per lane (element 2 lane + r in x_r).
__device__ __forceinline__ void warp_sort64(unsigned& x0, unsigned& x1, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 1) {
        const bool up = ((2 * lane) & k) == 0;
        const unsigned lo = min(x0, x1), hi = max(x0, x1);
        x0 = up ? lo : hi;
        x1 = up ? hi : lo;
      } else {
        const unsigned y0 = __shfl_xor_sync(0xffffffffu, x0, j >> 1);
        const unsigned y1 = __shfl_xor_sync(0xffffffffu, x1, j >> 1);
        const bool up = ((2 * lane) & k) == 0, low = ((2 * lane) & j) == 0;
        x0 = (low == up) ? min(x0, y0) : max(x0, y0);
        x1 = (low == up) ? min(x1, y1) : max(x1, y1);
      }
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1) attn_fwd_tc_kernel(
    const __grid_constant__ Geo g, const __grid_constant__ CUtensorMap tq128, const __grid_constant__ RunMaps km,
    const __grid_constant__ RunMaps vm, const float* __restrict__ pyrK, const float* __restrict__ pyrV,
    const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ o, float* __restrict__ lse, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const CUtensorMap* tk = km.m;
  const CUtensorMap* tv = vm.m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n1 = g.n[1], K1 = g.Kl[1];
  const int ngroups = (int)((int64_t)g.BH * n1 / QG);
  const int ntokens = ngroups / 2;            // n1 is a multiple of 16: a token's two groups lie in one slice
  const int stride = (int)gridDim.x;
  int nc = 0;                                 // pooled keys of levels >= 2 per token
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      ptx::mbar_init(&s.kfull[i], 1);
      ptx::mbar_init(&s.kempty[i], 1);
    }
    for (int i = 0; i < NMETA; ++i) {
      ptx::mbar_init(&s.mfull[i], 1);
      ptx::mbar_init(&s.mempty[i], META_ARRIVALS);
    }
    for (int i = 0; i < NQ; ++i) {
      ptx::mbar_init(&s.qfull[i], 1);
      ptx::mbar_init(&s.qempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.cfull[i], 1);
      ptx::mbar_init(&s.cempty[i], 1 + SOFT_WARPS);
      ptx::mbar_init(&s.s_full[i], 1);
      ptx::mbar_init(&s.s_empty[i], SOFT_WARPS);
      ptx::mbar_init(&s.p_full[i], SOFT_WARPS);
      ptx::mbar_init(&s.p_empty[i], 1);
      ptx::mbar_init(&s.o_full[i], 1);
      ptx::mbar_init(&s.o_empty[i], 4);
      ptx::mbar_init(&s.st_full[i], SOFT_WARPS);
    }
    for (int i = 0; i < 4; ++i) ptx::mbar_init(&s.xbar[i], PARTS);
    for (int i = 0; i < 2; ++i) ptx::mbar_init(&s.drain[i], 1);
    ptx::fence_mbar_init();
  }
  // Rows of absent key blocks in a partial chunk keep whatever the slot held;
  // start from zeros so that they are always finite.
  {
    uint4* z = reinterpret_cast<uint4*>(&s.slot[0]);
    const int n16 = (int)(sizeof(ChunkSlot) * NSLOT / 16);
    for (int e = threadIdx.x; e < n16; e += THREADS) z[e] = make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_proxy_async();
  }
  if (warp == 0) {
    tc::tmem_alloc(&s.tmem_base, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = s.tmem_base;
  // both O buffers start at zero (after each group the epilogue clears its buffer)
  if (warp >= EPI0 && warp < EPI0 + 4) {
    const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    uint32_t zero[16];
#pragma unroll
    for (int n = 0; n < 16; ++n) zero[n] = 0u;
#pragma unroll 1
    for (int q4 = 0; q4 < 8; ++q4) tc::tmem_st16(tl + COL_O + 16u * q4, zero);
    tc::tmem_wait_st();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // The CTA's groups: 2 t and 2 t + 1 for its tokens t = blockIdx.x + k * gridDim.x.
  const int my_tokens = (int)blockIdx.x < ntokens ? (ntokens - 1 - (int)blockIdx.x) / stride + 1 : 0;
  const uint32_t my_groups = 2u * (uint32_t)my_tokens;
  auto group_of = [&](uint32_t c) { return 2 * ((int)blockIdx.x + (int)(c >> 1) * stride) + (int)(c & 1); };

  if (warp == UNION_WARP) {
    // ============================================================ union
    uint32_t ent = 0, kc = 0, gc = 0;
    bool ok = true;
    // One entry into the ring; lanes e < nq hold block e in (ekb, em).  For a
    // chunk, each block's K / V row, and the TMA boxes: a run of consecutive
    // blocks (the union is ascending) is one box of up to RUNMAX blocks.
    auto put = [&](int kind, int gi, int nq, int flags, int ekb, int em) {
      const int ms = (int)(ent % NMETA);
      int good = 1;
      if (lane == 0) good = ptx::mbar_wait_bounded(&s.mempty[ms], ((ent / NMETA) & 1) ^ 1, kWaitLimitNs) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) {
        ok = false;
        if (lane == 0) report(err, 71);
        return;
      }
      Meta& M = s.meta[ms];
      const int box = run_box(ekb, nq, lane);
      if (lane < CK) {
        const int64_t bh = (int64_t)gi * QG / n1;
        M.msk[lane] = lane < nq ? em : 0;
        M.row[lane] = lane < nq ? (int)((bh * n1 + ekb) * 16) : 0;
        M.box[lane] = box;
      }
      if (lane == 0) {
        M.kind = kind;
        M.nq = nq;
        M.flags = flags;
        M.gc = (int)gc;
        M.tk = (int)(gc >> 1);
        M.kc = (int)kc;
        M.qrow = ((flags & kFirst) && gc + 1 < my_groups) ? group_of(gc + 1) * QG * 16 : -1;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.mfull[ms]);
      ++ent;
      if (kind == kChunk && nq > 0) ++kc;
    };
    // With at most 64 picks per group (K_1 <= 8) each lane holds two of the
    // next group's picks in registers, loaded while the current group merges.
    const bool small = QG * K1 <= 64;
    auto lists_of = [&](int gi) { return idx + g.idx_off[1] + (int64_t)gi * QG * K1; };
    int pf0 = 0, pf1 = 0;
    auto prefetch = [&](int gi) {
      if (!small || gi >= ngroups) return;
      const int32_t* gl = lists_of(gi);
      if (lane < QG * K1) pf0 = gl[lane];
      if (32 + lane < QG * K1) pf1 = gl[32 + lane];
    };
    // A token's pooled keys of levels >= 2 into coarse slot tk % 2.  Row r =
    // lane r: level l (rows ordered by level, K_l rows per enriched level
    // l >= 2), the r-th pick of the level-l list of the token's level-l
    // ancestor; all 16 vectors of a row in flight at once.
    const float bias_unit = log2f((float)g.B);
    auto build_coarse = [&](int t, uint32_t tk) {
      const int cs = (int)(tk & 1);
      int good = 1;
      if (lane == 0) good = ptx::mbar_wait_bounded(&s.cempty[cs], ((tk >> 1) & 1) ^ 1, kWaitLimitNs) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, good, 0)) {
        ok = false;
        if (lane == 0) report(err, 76);
        return;
      }
      const int bh = (2 * t * QG) / n1;
      const int a0 = 2 * t * QG - bh * n1;          // the token's first query block
      CoarseSlot& ct = s.crs[cs];
      int l = 0, tok = -1;
      int rr = lane;
      if (lane < nc) {
        for (int l2 = 2; l2 <= g.L; ++l2) {
          if (!((g.emask >> (l2 - 1)) & 1u)) continue;
          if (rr < g.Kl[l2]) {
            l = l2;
            break;
          }
          rr -= g.Kl[l2];
        }
        const int64_t grp = a0 / g.Bl[l - 1];
        const int v = idx[g.idx_off[l] + ((int64_t)bh * g.n[l] + grp) * g.Kl[l] + rr];
        tok = (v >= 0 && v < g.n[l]) ? v : -1;
      }
      ct.bias[lane] = tok >= 0 ? (float)l * bias_unit : -INFINITY;
      const int64_t off = tok >= 0 ? g.pyr_off[l] + ((int64_t)bh * g.n[l] + tok) * 64 : 0;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {   // K, then V
        const float4* src = reinterpret_cast<const float4*>((h == 0 ? pyrK : pyrV) + off);
        unsigned char* dst = h == 0 ? ct.k : ct.v;
        float4 x[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) x[c] = tok >= 0 ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          *reinterpret_cast<uint2*>(dst + ptx::sw128(lane, c * 4)) =
              make_uint2(ptx::pack_bf16(x[c].x, x[c].y), ptx::pack_bf16(x[c].z, x[c].w));
      }
      ptx::fence_proxy_async();   // the tile is read by the tensor cores
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.cfull[cs]);
    };
    prefetch(2 * (int)blockIdx.x);
    for (; gc < my_groups && ok; ++gc) {
      const int gi = group_of(gc);
      if ((gc & 1) == 0 && nc > 0) build_coarse(gi >> 1, gc >> 1);
      if (!ok) break;
      int flags = kFirst;
      if (nc > 0) {
        put(kCoarse, gi, 0, flags, 0, 0);
        flags = 0;
      }
      __syncwarp();
      if (small) {
        // at most 64 picks: sort (block << 3 | query block) keys, one run of
        // equal blocks per union entry, the run's query blocks as its mask
        const int np = QG * K1;
        auto key = [&](int v, int e) -> unsigned {
          return (e < np && v >= 0 && v < n1) ? ((unsigned)v << 3) | (unsigned)(e / K1) : 0xffffffffu;
        };
        unsigned x0 = key(pf0, lane), x1 = key(pf1, 32 + lane);
        if (gc + 1 < my_groups) prefetch(group_of(gc + 1));
        warp_sort64(x0, x1, lane);
        // element 2 lane (x0) and 2 lane + 1 (x1); a run has at most 8 elements
        const unsigned prev = __shfl_up_sync(0xffffffffu, x1, 1);
        const bool v0 = x0 != 0xffffffffu, v1 = x1 != 0xffffffffu;
        const bool f0 = v0 && (lane == 0 || (x0 >> 3) != (prev >> 3));
        const bool f1 = v1 && (x1 >> 3) != (x0 >> 3);
        unsigned m0 = 1u << (x0 & 7), m1 = 1u << (x1 & 7);
        if (v1 && (x1 >> 3) == (x0 >> 3)) m0 |= m1;
#pragma unroll
        for (int dl = 1; dl <= 4; ++dl) {
          const unsigned a = __shfl_down_sync(0xffffffffu, x0, dl), c = __shfl_down_sync(0xffffffffu, x1, dl);
          if (lane + dl < 32) {
            if (dl <= 3) {
              if (a != 0xffffffffu && (a >> 3) == (x0 >> 3)) m0 |= 1u << (a & 7);
              if (c != 0xffffffffu && (c >> 3) == (x0 >> 3)) m0 |= 1u << (c & 7);
            }
            if (a != 0xffffffffu && (a >> 3) == (x1 >> 3)) m1 |= 1u << (a & 7);
            if (dl <= 3 && c != 0xffffffffu && (c >> 3) == (x1 >> 3)) m1 |= 1u << (c & 7);
          }
        }
        const unsigned b0 = __ballot_sync(0xffffffffu, f0), b1 = __ballot_sync(0xffffffffu, f1);
        const unsigned lt = (1u << lane) - 1u;
        const int pos0 = __popc(b0 & lt) + __popc(b1 & lt);
        int* ukb = s.stage;
        int* umk = s.stage + 64;
        if (f0) {
          ukb[pos0] = (int)(x0 >> 3);
          umk[pos0] = (int)m0;
        }
        if (f1) {
          ukb[pos0 + (f0 ? 1 : 0)] = (int)(x1 >> 3);
          umk[pos0 + (f0 ? 1 : 0)] = (int)m1;
        }
        const int nu = __popc(b0) + __popc(b1);
        __syncwarp();
        for (int c0 = 0; c0 < nu && ok; c0 += CK) {
          const int nq = nu - c0 < CK ? nu - c0 : CK;
          put(kChunk, gi, nq, flags, lane < nq ? ukb[c0 + lane] : 0, lane < nq ? umk[c0 + lane] : 0);
          flags = 0;
        }
      } else {
        // merge the group's 8 ascending lists: lane j < 8 walks list j
        const int32_t* glists = lists_of(gi);
        const bool staged = QG * K1 <= STAGE;
        if (staged) {
          for (int e = lane; e < QG * K1; e += 32) s.stage[e] = glists[e];
          __syncwarp();
        }
        const int32_t* lists = staged ? s.stage : glists;
        int cur = lane < QG ? lane * K1 : 0;
        const int end = lane < QG ? (lane + 1) * K1 : 0;
        auto val = [&](int pos) -> unsigned {
          if (pos >= end) return kNone;
          const int a = lists[pos];
          return (a >= 0 && a < n1) ? (unsigned)a : kNone;   // an id outside its level ends the list
        };
        unsigned h = val(cur), hn = val(cur + 1);
        int cnt = 0, ekb = 0, em = 0;
        while (ok) {
          const unsigned kb = __reduce_min_sync(0xffffffffu, h);
          if (kb == kNone) break;
          const unsigned m = __ballot_sync(0xffffffffu, h == kb) & 0xffu;
          if (h == kb) {
            ++cur;
            h = hn;
            hn = val(cur + 1);
          }
          if (lane == (cnt & 7)) {
            ekb = (int)kb;
            em = (int)m;
          }
          ++cnt;
          if ((cnt & 7) == 0) {
            put(kChunk, gi, CK, flags, ekb, em);
            flags = 0;
          }
        }
        if (ok && (cnt & 7)) {
          put(kChunk, gi, cnt & 7, flags, ekb, em);
          flags = 0;
        }
      }
      if (ok) put(kGroupEnd, gi, 0, flags, 0, 0);
    }
    // the end marker, once for each producer (they take alternate entries)
    for (int p = 0; p < NPROD && ok; ++p) put(kEnd, 0, 0, 0, 0, 0);
  } else if (warp >= PRODUCER0 && warp < PRODUCER0 + NPROD) {
    // ============================================================ producers
    const int pw = warp - PRODUCER0;
    if (lane < kRunMax) {
      ptx::prefetch_tmap(&tk[lane]);
      ptx::prefetch_tmap(&tv[lane]);
    }
    if (lane == 0) ptx::prefetch_tmap(&tq128);
    bool ok = true;
    auto wait_lane0 = [&](uint64_t* bar, uint32_t parity, int code) {
      int good = 1;
      if (lane == 0) good = ptx::mbar_wait_bounded(bar, parity, kWaitLimitNs) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) {
        ok = false;
        if (lane == 0) report(err, code);
      }
    };
    // Q of the CTA's group c into slot c % NQ (its previous user, group c - NQ, is done)
    uint32_t qlast[NQ];
    int nql = 0;
    auto load_q = [&](uint32_t c, int row) {
      const int qs = (int)(c % NQ);
      wait_lane0(&s.qempty[qs], ((c / NQ) & 1) ^ 1, 72);
      if (!ok) return;
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(&s.qfull[qs], QG * 2048u);
        ptx::tma_load_2d(s.qs[qs].q, &tq128, 0, row, &s.qfull[qs]);
      }
      __syncwarp();
      qlast[nql % NQ] = c;
      ++nql;
    };
    if (pw == 0 && my_groups > 0) load_q(0, group_of(0) * QG * 16);
    uint32_t klast[NSLOT];
    int nkl = 0;
    for (uint32_t e = (uint32_t)pw; ok; e += NPROD) {
      const int ms = (int)(e % NMETA);
      wait_lane0(&s.mfull[ms], (e / NMETA) & 1, 73);
      if (!ok) break;
      const Meta& M = s.meta[ms];
      const int kind = M.kind, nq = M.nq, flags = M.flags, qrow = M.qrow;
      const uint32_t kc = (uint32_t)M.kc, gc = (uint32_t)M.gc;
      const int row = lane < CK ? M.row[lane] : 0;
      const int box = lane < CK ? M.box[lane] : 0;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.mempty[ms]);   // the entry is in registers
      if (kind == kEnd) break;
      if (kind == kChunk && nq > 0) {   // K and V into slot kc % NSLOT, one box per run
        const int ks = (int)(kc % NSLOT);
        wait_lane0(&s.kempty[ks], ((kc / NSLOT) & 1) ^ 1, 74);
        if (!ok) break;
        uint64_t* bar = &s.kfull[ks];
        if (lane == 0) ptx::mbar_arrive_expect_tx(bar, (uint32_t)nq * 4096u);
        __syncwarp();
        if (box > 0) {
          ptx::tma_load_2d(s.slot[ks].k + lane * 2048, &tk[box - 1], 0, row, bar);
          ptx::tma_load_2d(s.slot[ks].v + lane * 2048, &tv[box - 1], 0, row, bar);
        }
        __syncwarp();
        klast[nkl % NSLOT] = kc;
        ++nkl;
      }
      // the next group's Q as soon as this group starts
      if ((flags & kFirst) && qrow >= 0) load_q(gc + 1, qrow);
    }
    // After a timeout, do not leave while copies this warp issued may still be
    // landing.  (Otherwise the MMA warp has waited for every one of them; and
    // the other producer's later copies into the same slots advance their
    // barriers, so these waits would stall on a phase that never comes.)
    if (!ok && lane == 0) {
      for (int i = nkl > NSLOT ? nkl - NSLOT : 0; i < nkl; ++i) {
        const uint32_t c = klast[i % NSLOT];
        ptx::mbar_wait_bounded(&s.kfull[c % NSLOT], (c / NSLOT) & 1, kWaitLimitNs);
      }
      for (int i = nql > NQ ? nql - NQ : 0; i < nql; ++i) {
        const uint32_t c = qlast[i % NQ];
        ptx::mbar_wait_bounded(&s.qfull[c % NQ], (c / NQ) & 1, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == MMA_WARP || warp == PV_WARP) {
    // ============================================================ MMA issue
    // Two converged warps, one elected lane each: warp MMA_WARP issues every
    // S, warp PV_WARP every O update, so that S of entry i + 1 never waits
    // behind the issue of entry i's O update (which blocks while the tensor
    // pipe works through S).  Each reads every entry; commits track only the
    // issuing thread's MMAs.  Descriptors are built once and advanced by
    // adding to their start-address field (16-byte units, no carry: shared
    // addresses are below 256 KB).
    constexpr uint32_t idS = tc::idesc_bf16(128, 128, 0, 0);   // S: A = Q (K-major), B = K (K-major)
    constexpr uint32_t idSc = tc::idesc_bf16(128, 32, 0, 0);   // the same against the 32 pooled keys
    constexpr uint32_t idO = tc::idesc_bf16(128, 64, 0, 1);    // O += P V: A = P (TMEM), B = V (MN-major)
    constexpr uint64_t kSlotStep = sizeof(ChunkSlot) >> 4, kQStep = sizeof(QSlot) >> 4,
                       kCrsStep = sizeof(CoarseSlot) >> 4;
    const uint64_t dq0 = tc::sw128_desc(ptx::smem_u32(s.qs[0].q), 16, 1024);
    const uint64_t dk0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].k), 16, 1024);
    const uint64_t dv0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].v), 16, 1024);
    const uint64_t dck0 = tc::sw128_desc(ptx::smem_u32(s.crs[0].k), 16, 1024);
    const uint64_t dcv0 = tc::sw128_desc(ptx::smem_u32(s.crs[0].v), 16, 1024);
    const bool is_s = warp == MMA_WARP;
    bool ok = true;
    uint32_t seen = 0, sidx = 0;
    bool o_started = false;   // O update warp: the group has taken its O buffer
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok && !ptx::mbar_wait_bounded(bar, parity, kWaitLimitNs)) ok = false;
      return ok;
    };
    while (ok) {
      const int ms = (int)(seen % NMETA);
      if (!wait(&s.mfull[ms], (seen / NMETA) & 1)) break;
      const Meta& m = s.meta[ms];
      const int kind = m.kind, nq = m.nq, flags = m.flags;
      const uint32_t gc = (uint32_t)m.gc, tk = (uint32_t)m.tk, kc = (uint32_t)m.kc;
      __syncwarp();
      if (tc::elect_one()) ptx::mbar_arrive(&s.mempty[ms]);   // the entry is in registers
      __syncwarp();
      ++seen;
      if (kind == kEnd) break;
      const bool chunk = kind == kChunk && nq > 0;
      const bool has_s = kind == kCoarse || chunk;
      const uint32_t qs = gc % NQ, ob = gc & 1;
      if (is_s) {
        if (kind == kGroupEnd) {   // every S of the group has been issued: its Q is free once they finish
          if (tc::elect_one()) tc::commit(&s.qempty[qs]);
          __syncwarp();
          continue;
        }
        if ((flags & kFirst) && !wait(&s.qfull[qs], (gc / NQ) & 1)) break;   // the group's Q has landed
        if (kind == kCoarse && (gc & 1) == 0 && !wait(&s.cfull[tk & 1], (tk >> 1) & 1)) break;
        if (chunk && !wait(&s.kfull[kc % NSLOT], (kc / NSLOT) & 1)) break;
        if (!has_s) continue;
        const uint32_t b = sidx & 1, u = sidx >> 1;
        if (!wait(&s.s_empty[b], (u & 1) ^ 1)) break;   // the softmax warps have read S(b) of entry sidx - 2
        tc::fence_after_sync();
        const uint64_t go = kQStep * (uint64_t)qs;
        if (tc::elect_one()) {
          if (chunk) {
            const uint64_t so = kSlotStep * (uint64_t)(kc % NSLOT);
#pragma unroll
            for (int k = 0; k < 4; ++k)   // K steps of 16 channels: 32 bytes inside the 128-byte rows
              tc::mma_bf16(tbase + COL_S + 128u * b, dq0 + go + 2u * k, dk0 + so + 2u * k, idS, k > 0);
          } else {
            const uint64_t co = kCrsStep * (uint64_t)(tk & 1);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc::mma_bf16(tbase + COL_S + 128u * b, dq0 + go + 2u * k, dck0 + co + 2u * k, idSc, k > 0);
          }
          tc::commit(&s.s_full[b]);
        }
        __syncwarp();
        ++sidx;
      } else {
        if (has_s) {
          const uint32_t b = sidx & 1, u = sidx >> 1;
          if (!wait(&s.p_full[b], u & 1)) break;
          // the group's first O update: its last group's epilogue has read and cleared the buffer
          if (!o_started && !wait(&s.o_empty[ob], ((gc >> 1) & 1) ^ 1)) break;
          // V landed with K (the S warp saw it; the phase cannot have moved on
          // before this warp frees the slot)
          if (chunk && !wait(&s.kfull[kc % NSLOT], (kc / NSLOT) & 1)) break;
          tc::fence_after_sync();
          const uint32_t oc = tbase + COL_O + 64u * ob, pc = tbase + COL_P + 64u * b;
          if (tc::elect_one()) {
            if (chunk) {
              const uint64_t so = kSlotStep * (uint64_t)(kc % NSLOT);
#pragma unroll
              for (int k = 0; k < CK; ++k) {   // key block k: A 8 TMEM columns, B 2 KB
                if (k >= nq) break;
                tc::mma_bf16_ta(oc, pc + 8u * k, dv0 + so + 128u * k, idO, true);
              }
              tc::commit(&s.kempty[kc % NSLOT]);
            } else {
              const uint64_t co = kCrsStep * (uint64_t)(tk & 1);
#pragma unroll
              for (int k = 0; k < 2; ++k) tc::mma_bf16_ta(oc, pc + 8u * k, dcv0 + co + 128u * k, idO, true);
              if (gc & 1) tc::commit(&s.cempty[tk & 1]);
            }
            tc::commit(&s.p_empty[b]);
          }
          __syncwarp();
          o_started = true;
          ++sidx;
        } else if (kind == kGroupEnd) {
          // no O update in this group: still take the buffer over in order
          if (!o_started && !wait(&s.o_empty[ob], ((gc >> 1) & 1) ^ 1)) break;
          if (tc::elect_one()) tc::commit(&s.o_full[ob]);   // the group's O is complete
          __syncwarp();
          o_started = false;
        }
      }
    }
    if (!ok && lane == 0) report(err, is_s ? 77 : 75);
    // every MMA issued here has finished before TMEM is released
    if (tc::elect_one()) tc::commit(&s.drain[is_s ? 0 : 1]);
    __syncwarp();
    ptx::mbar_wait_bounded(&s.drain[is_s ? 0 : 1], 0, kWaitLimitNs);
  } else if (warp < SOFT_WARPS) {
    // ============================================================ softmax
    // The four warps w, w + 4, w + 8, w + 12 share TMEM lanes 32 (w % 4)..
    // (one query row per thread); part p = w / 4 takes key blocks 2 p, 2 p + 1
    // of a chunk, and parts 0 and 1 take pooled keys 0-15 and 16-31.  Per
    // entry each part finds its part of the row maximum, the four exchange it
    // through shared memory, and all take the same decision on the running
    // maximum.  Each keeps its own partial row sum.
    const int sub = warp & 3, part = warp >> 2;
    const int row = sub * 32 + lane;                    // query row of the group
    const int qbl = row >> 4;                           // its query block within the group
    const float log2B = log2f((float)g.B);
    const float sc2 = g.scale * kLog2e;                 // logits in the log2 domain
    const bool enrich1 = g.emask & 1u;
    const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
    uint32_t i = 0, sidx = 0;
    float m = -INFINITY, lsum = 0.f;
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity, int code) {
      if (ok && !ptx::mbar_wait_bounded(bar, parity, kWaitLimitNs)) {
        ok = false;
        report(err, code);
      }
      return ok;
    };
    while (ok) {
      const int ms = (int)(i % NMETA);
      if (!wait(&s.mfull[ms], (i / NMETA) & 1, 78)) break;
      const Meta& M = s.meta[ms];
      const int kind = M.kind, nq = M.nq;
      const uint32_t gc = (uint32_t)M.gc, tk = (uint32_t)M.tk;
      const int gs = (int)(gc & 1);
      unsigned pick = 0;                                // this row's picks among the part's 2 blocks
      if (kind == kChunk) {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * part + jj;
          if (j < nq) pick |= (((unsigned)M.msk[j] >> qbl) & 1u) << jj;
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.mempty[ms]);   // the entry is in registers
      ++i;
      if (kind == kEnd) break;
      if (kind == kGroupEnd) {
        // the epilogue has read this buffer's statistics of two groups ago
        if (!wait(&s.o_empty[gs], ((gc >> 1) & 1) ^ 1, 78)) break;
        if (part == 0) s.stat_m[gs][row] = m;
        s.stat_l[gs][part][row] = lsum;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&s.st_full[gs]);
        m = -INFINITY;
        lsum = 0.f;
        continue;
      }
      if (kind == kChunk && nq == 0) continue;
      const bool coarse = kind == kCoarse;
      const uint32_t b = sidx & 1, u = sidx >> 1;
      const uint32_t sc = COL_S + 128u * b, pcol = COL_P + 64u * b, oc = COL_O + 64u * (uint32_t)gs;
      if (!wait(&s.s_full[b], u & 1, 79)) break;
      tc::fence_after_sync();
      // the tile's bias row came from the union warp: observe its barrier too
      if (coarse && gs == 0 && !wait(&s.cfull[tk & 1], (tk >> 1) & 1, 79)) break;
      const float* bias = s.crs[tk & 1].bias + 16 * part;
      // blocks of 16 columns this warp reads: its 2 key blocks, or its 16 pooled keys
      const int nblk = coarse ? (part < 2 ? 1 : 0) : 2;
      const unsigned need = coarse ? (unsigned)nblk : __reduce_or_sync(0xffffffffu, pick);
      const unsigned mine = coarse ? need : pick;
      const uint32_t scol0 = sc + (coarse ? 16u : 32u) * (uint32_t)part;
      const uint32_t pcol0 = pcol + (coarse ? 8u : 16u) * (uint32_t)part;
      // the part's row maximum over the keys this row attends
      float mx = -INFINITY;
#pragma unroll 1
      for (int jj = 0; jj < nblk; ++jj) {
        if (!((need >> jj) & 1u)) continue;
        uint32_t sr[16];
        tc::tmem_ld16(tl + scol0 + 16u * jj, sr);
        tc::tmem_wait_ld();
        if (!((mine >> jj) & 1u)) continue;
        float bm = -INFINITY, zs = 0.f;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          const float zz = coarse ? fmaf(__uint_as_float(sr[n]), sc2, bias[n]) : __uint_as_float(sr[n]);
          bm = fmaxf(bm, zz);
          zs += zz;
        }
        if (!coarse) {
          bm *= sc2;
          if (enrich1) bm = fmaxf(bm, fmaf(zs * (1.f / 16.f), sc2, log2B));   // the block's pooled level-1 token
        }
        mx = fmaxf(mx, bm);
      }
      // exchange with the other parts (by entry parity, so that a slow partner
      // still reads this entry's values)
      s.xmax[sidx & 1][part][row] = mx;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.xbar[sub]);
      if (!wait(&s.xbar[sub], sidx & 1, 79)) break;
#pragma unroll
      for (int p = 0; p < PARTS; ++p) mx = fmaxf(mx, s.xmax[sidx & 1][p][row]);
      const float mn = fmaxf(m, mx);
      bool resc = false;
      float a = 1.f;
      if (m == -INFINITY) {
        m = mn;
      } else if (mn > m + kHeadroom) {
        resc = true;
        a = ptx::ex2(m - mn);
        m = mn;
        lsum *= a;
      }
      if (part == 0 && __any_sync(0xffffffffu, resc)) {   // O holds every earlier update (entry sidx - 1): scale it
        if (!wait(&s.p_empty[(sidx - 1) & 1], ((sidx - 1) >> 1) & 1, 79)) break;
        tc::fence_after_sync();
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t r[16];
          tc::tmem_ld16(tl + oc + 16u * q4, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < 16; ++n) r[n] = __float_as_uint(__uint_as_float(r[n]) * a);
          tc::tmem_st16(tl + oc + 16u * q4, r);
        }
        tc::tmem_wait_st();
      }
      if (!wait(&s.p_empty[b], (u & 1) ^ 1, 79)) break;   // the O update of entry sidx - 2 has read P(b)
      tc::fence_after_sync();
      // P of the blocks this row picked (plus the block's pooled-token share),
      // zero for the blocks it did not pick (the O update takes every row)
#pragma unroll 1
      for (int jj = 0; jj < nblk; ++jj) {
        uint32_t pw[8];
        if (!((need >> jj) & 1u)) {
#pragma unroll
          for (int n = 0; n < 8; ++n) pw[n] = 0u;
          tc::tmem_st8(tl + pcol0 + 8u * jj, pw);
          continue;
        }
        uint32_t sr[16];
        tc::tmem_ld16(tl + scol0 + 16u * jj, sr);
        tc::tmem_wait_ld();
        if ((mine >> jj) & 1u) {
          float sh = 0.f;
          if (!coarse && enrich1) {
            float zs = 0.f;
#pragma unroll
            for (int n = 0; n < 16; ++n) zs += __uint_as_float(sr[n]);
            const float pc = ptx::ex2(fmaf(zs * (1.f / 16.f), sc2, log2B) - m);
            lsum += pc;
            sh = pc * (1.f / 16.f);
          }
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            float p0, p1;
            if (coarse) {
              const float z0 = fmaf(__uint_as_float(sr[2 * n]), sc2, bias[2 * n]);
              const float z1 = fmaf(__uint_as_float(sr[2 * n + 1]), sc2, bias[2 * n + 1]);
              p0 = z0 == -INFINITY ? 0.f : ptx::ex2(z0 - m);
              p1 = z1 == -INFINITY ? 0.f : ptx::ex2(z1 - m);
            } else {
              p0 = ptx::ex2(fmaf(__uint_as_float(sr[2 * n]), sc2, -m));
              p1 = ptx::ex2(fmaf(__uint_as_float(sr[2 * n + 1]), sc2, -m));
            }
            lsum += p0 + p1;
            pw[n] = ptx::pack_bf16(p0 + sh, p1 + sh);
          }
        } else {
#pragma unroll
          for (int n = 0; n < 8; ++n) pw[n] = 0u;
        }
        tc::tmem_st8(tl + pcol0 + 8u * jj, pw);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&s.s_empty[b]);
        ptx::mbar_arrive(&s.p_full[b]);
        if (coarse && gs == 1) ptx::mbar_arrive(&s.cempty[tk & 1]);   // done with the tile's biases
      }
      ++sidx;
    }
  } else {
    // ============================================================ epilogue
    const int sub = warp - EPI0;                        // == warp % 4, the TMEM subpartition this warp may read
    const int row = sub * 32 + lane;
    const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
    uint32_t zero[16];
#pragma unroll
    for (int n = 0; n < 16; ++n) zero[n] = 0u;
    for (uint32_t gc = 0; gc < my_groups; ++gc) {
      const int gs = (int)(gc & 1);
      if (!ptx::mbar_wait_bounded(&s.o_full[gs], (gc >> 1) & 1, kWaitLimitNs) ||
          !ptx::mbar_wait_bounded(&s.st_full[gs], (gc >> 1) & 1, kWaitLimitNs)) {
        report(err, 80);
        break;
      }
      tc::fence_after_sync();
      const float mrow = s.stat_m[gs][row];
      float lrow = 0.f;
#pragma unroll
      for (int p = 0; p < PARTS; ++p) lrow += s.stat_l[gs][p][row];
      const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
      const int64_t grow = (int64_t)group_of(gc) * QG * 16 + row;
      uint4* drow = reinterpret_cast<uint4*>(o + grow * 64);
      const uint32_t oc = tl + COL_O + 64u * (uint32_t)gs;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t r[16];
        tc::tmem_ld16(oc + 16u * q4, r);
        tc::tmem_wait_ld();
        tc::tmem_st16(oc + 16u * q4, zero);           // cleared for the buffer's next group
        uint32_t w[8];
#pragma unroll
        for (int n = 0; n < 8; ++n)
          w[n] = ptx::pack_bf16(__uint_as_float(r[2 * n]) * inv, __uint_as_float(r[2 * n + 1]) * inv);
        drow[2 * q4] = make_uint4(w[0], w[1], w[2], w[3]);
        drow[2 * q4 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      tc::tmem_wait_st();
      lse[grow] = lrow > 0.f ? (mrow + log2f(lrow)) * kLn2 : -INFINITY;
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.o_empty[gs]);
    }
  }

  // ------------------------------------------------------------ teardown
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, TMEM_COLS);
  }
}

}  // namespace fwdtc

// Largest level-1 list the tensor-core forward takes (the K = all lists of a
// 256 x 256 image); longer lists go to the CUDA-core kernel.
constexpr int kFwdMaxK1 = 4096;

bool attn_fwd_mma_supported(const Geo& g) {
  if (!g.bf16 || g.d != 64 || g.B != 16) return false;
  if (g.n[1] % 16) return false;              // whole level-2 tokens: two groups of 8 query blocks
  if (g.Kl[1] < 1 || g.Kl[1] > kFwdMaxK1) return false;
  if (g.n[1] >= (1 << 23)) return false;      // union keys pack (block << 3) | query block into 32 bits
  int nc = 0;
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];
  if (nc > fwdtc::COARSE) return false;
  if ((int64_t)g.BH * g.N >= (1ll << 31)) return false;
  if ((int64_t)g.BH * g.n[1] * g.Kl[1] >= (1ll << 31)) return false;
  return true;
}

cudaError_t launch_attn_fwd_mma(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                                const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  CUtensorMap tq128;
  RunMaps km, vm;
  cudaError_t e = make_token_map_box(&tq128, q, rows, fwdtc::QG * 16);
  if (e == cudaSuccess) e = make_run_maps(&km, k, rows);
  if (e == cudaSuccess) e = make_run_maps(&vm, v, rows);
  if (e != cudaSuccess) return e;
  const int ntokens = (int)((int64_t)g.BH * g.n[1] / (2 * fwdtc::QG));
  if (ntokens == 0) return cudaSuccess;
  const size_t smem = sizeof(fwdtc::Smem) + 1024;
  e = cudaFuncSetAttribute(fwdtc::attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = ntokens < sms ? ntokens : sms;
  fwdtc::attn_fwd_tc_kernel<<<grid, fwdtc::THREADS, smem, s>>>(g, tq128, km, vm, pyrK, pyrV, idx,
                                                               (__nv_bfloat16*)o, lse, device_error_word());
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace llsa
