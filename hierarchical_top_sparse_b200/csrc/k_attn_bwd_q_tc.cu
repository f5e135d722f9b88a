// k_attn_bwd_q_tc.cu -- query-major pass of the sparse attention backward on
// the 5th-generation tensor cores (tcgen05, accumulators in tensor memory),
// bf16, d = 64, B = 16 (Trainable Log-linear Sparse Attention summary §4.1).
//
// Work unit: a level-2 token, two query groups of 8 sibling query blocks
// (128 queries each).  The key blocks that any block of a group picked (the
// union of the 8 pick lists, each with an 8-bit mask of which query blocks
// picked it) are taken 8 at a time: a chunk of 128 keys whose K and V tiles
// TMA stacks into 128-row, 128-byte-swizzled operands.  Per chunk:
//   S = Q_G K_c^T and dP = dO_G V_c^T          (M = 128 queries, N = 128 keys, K = 64)
//   one thread per (query row, pair of key blocks) reads its S and dP values
//   from TMEM and, for the blocks its query block picked, forms
//   dS = P (dP - D) with P = exp(z - LSE), plus the block's pooled level-1
//   token (mean logit + ln B, mean dP) folded in as dS_c / B on each of the
//   block's 16 keys (hierarchical KV enrichment, §四); other blocks get zeros;
//   dQ += dS K_c                               (M = 128 queries, N = 64, K = 128 keys)
// accumulated in TMEM over the group's chunks, with dS itself written to TMEM
// by the softmax warps (tcgen05.st) and read from there as the A operand, so
// that only K_c comes from shared memory.  The pooled keys of levels >= 2
// are the same for the token's 256 queries: after the union chunks each group
// runs one more chunk against them (logit bias ln B^l), adds dS_c Kc to dQ and
// accumulates their gradients dS_c^T Q and P_c^T dO in TMEM over the token, so
// each pooled key gets one fp32 reduction per 4 channels and token.
//
// A pre-pass, q_prep_kernel (one CTA per token), writes what does not need
// the tensor cores: the unions (each entry (key block << 8) | mask, ascending,
// in the group's own range of the level-1 index layout), D = rowsum(dO * O)
// of every query row, and each token's pooled-key tile (bf16 K / V rows in
// the swizzled operand layout, bias, level, id).
//
// Warp roles of the main kernel, one CTA per SM (22 warps):
//   * warp 20, producer: claims tokens one at a time from a counter that all
//     CTAs share (and hands their ids to the epilogue warps), loads each
//     group's Q and dO (one 128-row TMA box each) into one of two group
//     slots, the token's pooled-key tile (one bulk copy) into one of two
//     coarse slots, and the K/V tiles of each union chunk (one lane per 2 KB
//     tile) into one of NSLOT chunk slots, and puts one entry per chunk (and
//     one closing entry per group) on the chunk ring;
//   * warp 21, MMA: a converged warp whose elected lane issues every MMA,
//     the S / dP of chunk i + 1 ahead of the dQ of chunk i;
//   * warps 0-15, softmax: warps w, w + 4, w + 8, w + 12 share TMEM lanes
//     32 (w % 4).. and take key blocks 2 (w / 4), 2 (w / 4) + 1 of a chunk;
//     each thread reads its row's LSE and D from global memory at the
//     group's first entry;
//   * warps 16-19, epilogue: dQ out of TMEM, and the pooled-key gradients'
//     reductions.
// Every hand-off is an mbarrier, every wait is bounded; on a timeout the
// kernel sets the device error word and stops.
#include <math.h>
#include <stddef.h>

#include "llsa_internal.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {
namespace bwdq {

constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int QG = 8;               // query blocks per group (128 queries)
constexpr int CK = 8;               // key blocks per chunk (128 keys)
constexpr int NSLOT = 3;            // chunk slots
constexpr int COARSE = 32;          // pooled keys of levels >= 2 per token, at most
constexpr int SOFT_WARPS = 16, EPI_WARP0 = 16, PRODUCER_WARP = 20, MMA_WARP = 21;
constexpr int THREADS = 22 * 32;
constexpr uint32_t TMEM_COLS = 512;
// S 0-127, dP 128-255, dQ 256-319, dS of a chunk 320-383 (bf16 pairs: the A
// operand of dQ += dS K), pooled-key gradients dK 384-447 and dV 448-511
// ([pooled key][channel], M = 64: pooled key 16 w + i in TMEM lane 32 w + i)
constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DQ = 256, COL_DS = 320, COL_GK = 384, COL_GV = 448;
enum : int { kEnd = 0, kChunk = 1, kTail = 2 };
constexpr int kFirst = 1;           // first entry of a group
constexpr int EMPTY_ARRIVALS = 1 + SOFT_WARPS;   // a chunk slot is freed by the MMA thread and every softmax warp
constexpr int TRING = 4;            // token ids in flight between the producer and the epilogue

struct ChunkSlot {
  alignas(1024) unsigned char k[CK * 2048];    // [128 keys][64] bf16, 128-byte swizzle
  alignas(1024) unsigned char v[CK * 2048];
};

struct GroupSlot {
  alignas(1024) unsigned char q[QG * 2048];    // [128 queries][64] bf16, 128-byte swizzle
  alignas(1024) unsigned char dO[QG * 2048];
};

// A token's pooled keys of levels >= 2, as the pre-pass writes them to the
// workspace and one bulk copy brings them into shared memory (whose 1024-byte
// alignment makes the stored swizzle the one the MMA reads).
struct CoarseTile {
  unsigned char k[COARSE * 128];               // [32 pooled keys][64] bf16, 128-byte swizzle
  unsigned char v[COARSE * 128];
  float bias[COARSE];                          // logit bias (log2 domain); -inf: no key
  int level[COARSE];
  int tok[COARSE];                             // pooled token id, -1: none
};
static_assert(sizeof(CoarseTile) == kBwdCoarseTileBytes, "the workspace holds one CoarseTile per token");
static_assert(sizeof(CoarseTile) % 16 == 0, "bulk copies move multiples of 16 bytes");

struct alignas(1024) CoarseSlot {
  CoarseTile t;
};

struct Meta {
  int kind, gi, gs, nq, flags;                 // group, group slot, key blocks in the chunk
  int kb[CK];                                  // the chunk's key blocks (ids within the slice)
  int msk[CK];                                 // bit j: query block 8 g + j picked the key block
};

struct Smem {
  ChunkSlot slot[NSLOT];
  GroupSlot grp[2];
  CoarseSlot crs[2];
  // dS as the A operand of dQ += dS K: [query][key], keys contiguous
  // (K-major), 128-byte swizzle; keys 0-63 and 64-127 are two 16 KB halves.
  // The pooled-key chunk uses half 0 for dS_c and half 1 for P_c.
  alignas(1024) unsigned char sbuf[2 * 16384];
  Meta meta[NSLOT];
  alignas(8) uint64_t full[NSLOT], empty[NSLOT];
  uint64_t gfull[2], gempty[2];                // group slots: producer -> MMA, MMA -> producer
  uint64_t cfull[2], cempty[2];                // pooled-key tiles: producer -> MMA, MMA + epilogue (4 warps) -> producer
  uint64_t s_full, s_empty;                    // S / dP in TMEM: MMA -> softmax, softmax (16 warps) -> MMA
  uint64_t p_full, p_empty;                    // dS operand: softmax (16 warps) -> MMA, MMA -> softmax
  uint64_t acc_full, acc_empty;                // dQ of a group (phase = the CTA's group count): MMA -> epilogue, epilogue (4 warps) -> MMA
  uint64_t cacc_full, cacc_empty;              // pooled-key gradients: MMA -> epilogue, epilogue (4 warps) -> MMA
  uint64_t tid_full[TRING], tid_empty[TRING];  // the CTA's tokens in claim order: producer -> epilogue
  uint64_t drain;
  int tid[TRING];
  uint32_t tmem_base;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA exceeds the 227 KB limit");
static_assert(sizeof(ChunkSlot) % 1024 == 0 && sizeof(GroupSlot) % 1024 == 0 && sizeof(CoarseSlot) % 1024 == 0,
              "operands are addressed with fixed strides");

__device__ __forceinline__ void report(int* err, int code) {
  if (err) atomicExch(err, code);
}

// One warp: the union of query group gi's 8 level-1 pick lists (each sorted
// ascending), in ascending order, each entry (key block << 8) | mask where bit
// j says that query block 8 gi + j picked the key block.  Written at the
// group's own range of the level-1 index layout (8 K_1 slots); its size in
// ucount[gi].
// The lists are first staged in `stage` (UNION_STAGE words) when they fit,
// so that the merge loop reads shared memory rather than a chain of
// dependent global loads.
constexpr int UNION_STAGE = 512;
__device__ __forceinline__ void group_union(const Geo& g, const int32_t* __restrict__ idx,
                                            int32_t* __restrict__ ulist, int32_t* __restrict__ ucount, int gi,
                                            int lane, int* stage) {
  const int n1 = g.n[1], K1 = g.Kl[1];
  const int32_t* glists = idx + g.idx_off[1] + (int64_t)gi * QG * K1;   // the group's 8 consecutive lists
  const bool staged = QG * K1 <= UNION_STAGE;
  if (staged) {
    for (int e = lane; e < QG * K1; e += 32) stage[e] = glists[e];
    __syncwarp();
  }
  const int32_t* lists = staged ? stage : glists;
  int32_t* out = ulist + (int64_t)gi * QG * K1;
  // lane j < 8 walks list j
  int cur = lane < QG ? lane * K1 : 0;
  const int end = lane < QG ? (lane + 1) * K1 : 0;
  auto head = [&]() -> int {
    while (cur < end) {
      const int a = lists[cur];
      if (a >= 0 && a < n1) return a;
      ++cur;   // an id outside its level: skipped
    }
    return 0x7fffffff;
  };
  int h = head();
  int count = 0, val = 0;
  while (true) {
    const int kb = (int)__reduce_min_sync(0xffffffffu, (unsigned)h);
    if (kb == 0x7fffffff) break;
    const unsigned msk = __ballot_sync(0xffffffffu, h == kb) & 0xffu;
    if (h == kb) {
      ++cur;
      h = head();
    }
    if (lane == (count & 31)) val = (kb << 8) | (int)msk;
    ++count;
    if ((count & 31) == 0) out[count - 32 + lane] = val;   // 32 at a time, coalesced
  }
  if (lane < (count & 31)) out[(count & ~31) + lane] = val;
  if (lane == 0) ucount[gi] = count;
}

// One warp: the union of key group gi's 8 level-1 CSC lists (each sorted
// ascending), in ascending order, each entry (query block << 8) | mask where
// bit j says that the query block picked key block 8 gi + j.  Written at the
// group's own CSC range [offs(8 gi), offs(8 gi) + size) of ulist; its size in
// ucount[gi].  For the key-major pass.
__device__ __forceinline__ void key_group_union(const Geo& g, const int32_t* __restrict__ offs,
                                                const int32_t* __restrict__ qlist, int32_t* __restrict__ ulist,
                                                int32_t* __restrict__ ucount, int gi, int lane, int* stage) {
  constexpr int KG = 8;
  const int n1 = g.n[1];
  const int64_t slice_entries = (int64_t)n1 * g.Kl[1];
  const int bh = gi * KG / n1;
  const int kb0 = gi * KG - bh * n1;
  const int ow = lane <= KG ? offs[g.offs_off[1] + (int64_t)bh * (n1 + 1) + kb0 + lane] : 0;
  const int lo = __shfl_sync(0xffffffffu, ow, 0);
  const int hi = __shfl_sync(0xffffffffu, ow, KG);
  if (lo < 0 || hi < lo || (int64_t)hi > slice_entries) {   // never produced by the transpose
    if (lane == 0) ucount[gi] = 0;
    return;
  }
  const int32_t* slist = qlist + g.idx_off[1] + (int64_t)bh * slice_entries;
  int32_t* out = ulist + (int64_t)bh * slice_entries + lo;
  const bool staged = hi - lo <= UNION_STAGE;
  if (staged) {
    for (int e = lane; e < hi - lo; e += 32) stage[e] = slist[lo + e];
    __syncwarp();
  }
  // lane j < 8 walks list j
  int cur = __shfl_sync(0xffffffffu, ow, lane & 7);
  int end = __shfl_sync(0xffffffffu, ow, (lane & 7) + 1);
  if (lane >= KG || cur < lo || end < cur || end > hi) cur = end = 0;
  auto head = [&]() -> int {
    while (cur < end) {
      const int a = staged ? stage[cur - lo] : slist[cur];
      if (a >= 0 && a < n1) return a;
      ++cur;   // an id outside its level: skipped
    }
    return 0x7fffffff;
  };
  int h = head();
  int count = 0, val = 0;
  while (true) {
    const int q = (int)__reduce_min_sync(0xffffffffu, (unsigned)h);
    if (q == 0x7fffffff) break;
    const unsigned msk = __ballot_sync(0xffffffffu, h == q) & 0xffu;
    if (h == q) {
      ++cur;
      h = head();
    }
    if (lane == (count & 31)) val = (q << 8) | (int)msk;
    ++count;
    if ((count & 31) == 0) out[count - 32 + lane] = val;   // 32 at a time, coalesced
  }
  if (lane < (count & 31)) out[(count & ~31) + lane] = val;
  if (lane == 0) ucount[gi] = count;
}

constexpr int PREP_THREADS = 256;

// Pre-pass, two CTAs per level-2 token t (query groups 2t, 2t + 1; key groups
// 2t, 2t + 1 are the same 16 blocks as keys), the first doing the lists and
// the tile, the second D:
//   * warps 0, 1: the unions of the two query groups' pick lists;
//   * warps 2, 3: the unions of the two key groups' CSC lists (for the
//     key-major pass);
//   * D = rowsum(dO * O) of the token's 256 query rows (8 lanes per row);
//   * the token's tile of pooled keys of levels >= 2: the lists of level l
//     belong to the level-(l-1) ancestor of the token's query blocks; each
//     picked pooled K / V row converted to bf16 at its swizzled place, with
//     logit bias l ln B (log2 domain), its level and its id.
__global__ void __launch_bounds__(PREP_THREADS) q_prep_kernel(Geo g, const int32_t* __restrict__ idx,
                                                              const __nv_bfloat16* __restrict__ o,
                                                              const __nv_bfloat16* __restrict__ dO,
                                                              const float* __restrict__ pyrK,
                                                              const float* __restrict__ pyrV,
                                                              const int32_t* __restrict__ offs,
                                                              const int32_t* __restrict__ qlist,
                                                              int32_t* __restrict__ ulist, int32_t* __restrict__ ucount,
                                                              int32_t* __restrict__ ulist_kv,
                                                              int32_t* __restrict__ ucount_kv,
                                                              float* __restrict__ Dws, unsigned char* __restrict__ ctile,
                                                              int nc) {
  __shared__ int stage[4][UNION_STAGE];
  // Two blocks per token, interleaved: the odd one streams D (bound by DRAM),
  // the even one merges the unions and builds the pooled-key tile (bound by
  // latency), so that neither holds the other's resources.
  const int t = blockIdx.x >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x & 1) {
  const int64_t row0 = (int64_t)t * 2 * QG * 16;
#pragma unroll 2
  for (int it = 0; it < 8; ++it) {
    const int64_t gr = row0 + warp * 32 + it * 4 + (lane >> 3);
    const uint4 ov = reinterpret_cast<const uint4*>(o + gr * 64)[lane & 7];
    const uint4 gv = reinterpret_cast<const uint4*>(dO + gr * 64)[lane & 7];
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = __bfloat1622float2(o2[e]), b = __bfloat1622float2(g2[e]);
      acc = fmaf(a.x, b.x, acc);
      acc = fmaf(a.y, b.y, acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if ((lane & 7) == 0) Dws[gr] = acc;
  }
  return;
  }
  if (warp < 2) group_union(g, idx, ulist, ucount, 2 * t + warp, lane, stage[warp]);
  else if (warp < 4) key_group_union(g, offs, qlist, ulist_kv, ucount_kv, 2 * t + warp - 2, lane, stage[warp]);
  if (nc <= 0) return;
  const int n1 = g.n[1];
  const int bh = (2 * t * QG) / n1;
  const int a0 = 2 * t * QG - bh * n1;                // the token's first query block
  CoarseTile& ct = *reinterpret_cast<CoarseTile*>(ctile + (size_t)t * sizeof(CoarseTile));
  const float bias_unit = log2f((float)g.B);          // ln B in the log2 domain
  for (int e = threadIdx.x; e < COARSE * 16; e += PREP_THREADS) {
    const int r = e >> 4, chunk = e & 15;
    int l = 0, tok = -1;
    if (r < nc) {
      int rr = r;
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
    float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
    if (tok >= 0) {
      const int64_t off = g.pyr_off[l] + ((int64_t)bh * g.n[l] + tok) * 64 + chunk * 4;
      kv = *reinterpret_cast<const float4*>(pyrK + off);
      vv = *reinterpret_cast<const float4*>(pyrV + off);
    }
    const uint32_t o2 = ptx::sw128(r, chunk * 4);
    *reinterpret_cast<uint2*>(ct.k + o2) = make_uint2(ptx::pack_bf16(kv.x, kv.y), ptx::pack_bf16(kv.z, kv.w));
    *reinterpret_cast<uint2*>(ct.v + o2) = make_uint2(ptx::pack_bf16(vv.x, vv.y), ptx::pack_bf16(vv.z, vv.w));
    if (chunk == 0) {
      ct.bias[r] = tok >= 0 ? (float)l * bias_unit : -INFINITY;
      ct.level[r] = l;
      ct.tok[r] = tok;
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1) attn_bwd_q_tc_kernel(
    const __grid_constant__ Geo g, const __grid_constant__ CUtensorMap tq128, const __grid_constant__ CUtensorMap tdo128,
    const __grid_constant__ RunMaps tk, const __grid_constant__ RunMaps tv, const float* __restrict__ lse,
    const float* __restrict__ Dws, const int32_t* __restrict__ ulist, const int32_t* __restrict__ ucount,
    const unsigned char* __restrict__ ctile, __nv_bfloat16* __restrict__ dq, float* __restrict__ dPK,
    float* __restrict__ dPV, int* __restrict__ counter, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n1 = g.n[1], K1 = g.Kl[1];
  const int ngroups = (int)((int64_t)g.BH * n1 / QG);
  const int ntokens = ngroups / 2;            // n1 is a multiple of 16: a token's two groups lie in one slice
  int nc = 0;                                 // pooled keys of levels >= 2 per token
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], EMPTY_ARRIVALS);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.gfull[i], 1);
      ptx::mbar_init(&s.gempty[i], 1);
      ptx::mbar_init(&s.cfull[i], 1);
      ptx::mbar_init(&s.cempty[i], 1 + 4);
    }
    ptx::mbar_init(&s.s_full, 1);
    ptx::mbar_init(&s.s_empty, SOFT_WARPS);
    ptx::mbar_init(&s.p_full, SOFT_WARPS);
    ptx::mbar_init(&s.p_empty, 1);
    ptx::mbar_init(&s.acc_full, 1);
    ptx::mbar_init(&s.acc_empty, 4);
    ptx::mbar_init(&s.cacc_full, 1);
    ptx::mbar_init(&s.cacc_empty, 4);
    for (int i = 0; i < TRING; ++i) {
      ptx::mbar_init(&s.tid_full[i], 1);
      ptx::mbar_init(&s.tid_empty[i], 4);
    }
    ptx::mbar_init(&s.drain, 1);
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

  if (warp == PRODUCER_WARP) {
    // ============================================================ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tq128);
      ptx::prefetch_tmap(&tdo128);
    }
    if (lane < kRunMax) {
      ptx::prefetch_tmap(&tk.m[lane]);
      ptx::prefetch_tmap(&tv.m[lane]);
    }
    uint32_t issued = 0;
    bool ok = true;
    auto wait_free = [&](uint64_t* bar, uint32_t parity, int code) {
      int good = 1;
      if (lane == 0) good = ptx::mbar_wait_bounded(bar, parity, kWaitLimitNs) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) {
        ok = false;
        if (lane == 0) report(err, 51);
      }
    };
    // One ring entry: a chunk of nq key blocks (lane j < nq holds block j and
    // its mask in ek / em) or a group's closing entry.  A run of consecutive
    // key blocks is one box of up to four tiles: lane j issues the K box that
    // starts at block j, lane 8 + j the V box.
    auto emit = [&](int kind, int gi, int gs, int64_t bh, int nq, int flags, int ek, int em) {
      const int slot = (int)(issued % NSLOT);
      wait_free(&s.empty[slot], ((issued / NSLOT) & 1) ^ 1, 51);
      if (!ok) return;
      Meta& m = s.meta[slot];
      if (lane < nq) {
        m.kb[lane] = ek;
        m.msk[lane] = em;
      }
      __syncwarp();
      uint64_t* bar = &s.full[slot];
      if (lane == 0) {
        m.kind = kind;
        m.gi = gi;
        m.gs = gs;
        m.nq = nq;
        m.flags = flags;
        if (nq > 0)
          ptx::mbar_arrive_expect_tx(bar, (uint32_t)nq * 4096u);
        else
          ptx::mbar_arrive(bar);
      }
      __syncwarp();
      const int j = lane & 7;
      const int kj = __shfl_sync(0xffffffffu, ek, j);
      const int box = __shfl_sync(0xffffffffu, run_box(ek, nq, lane), j);
      if (lane < 16 && box > 0) {
        const int row = (int)((bh * n1 + kj) * 16);
        ChunkSlot& cs = s.slot[slot];
        if (lane < 8)
          ptx::tma_load_2d(cs.k + j * 2048, &tk.m[box - 1], 0, row, bar);
        else
          ptx::tma_load_2d(cs.v + j * 2048, &tv.m[box - 1], 0, row, bar);
      }
      __syncwarp();
      ++issued;
    };

    // Tokens are claimed one at a time from a counter that all CTAs share,
    // and handed to the epilogue warps in claim order (-1: no more).
    auto announce = [&](uint32_t k, int t) {
      const int r = (int)(k % TRING);
      wait_free(&s.tid_empty[r], ((k / TRING) & 1) ^ 1, 50);
      if (!ok) return;
      if (lane == 0) {
        s.tid[r] = t;
        ptx::mbar_arrive(&s.tid_full[r]);
      }
      __syncwarp();
    };
    auto claim = [&]() -> int {
      int v = 0;
      if (lane == 0) v = atomicAdd(counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    uint32_t tk_n = 0;   // tokens done by this CTA
    for (int t = claim(); t < ntokens && ok; t = claim(), ++tk_n) {
      announce(tk_n, t);
      if (!ok) break;
      // the token's two groups: counts and first 64 union entries, then Q / dO
      int cnt[2], e0[2], e1[2];
#pragma unroll
      for (int gs = 0; gs < 2; ++gs) {
        const int gi = 2 * t + gs;
        const int32_t* ul = ulist + (int64_t)gi * QG * K1;
        cnt[gs] = ucount[gi];
        e0[gs] = lane < cnt[gs] ? ul[lane] : 0;
        e1[gs] = 32 + lane < cnt[gs] ? ul[32 + lane] : 0;
      }
      // A group's Q / dO slot is freed when the MMA warp finishes the group,
      // and that MMA warp reads one ring entry ahead: so group 1's slot is
      // waited for only after group 0's first entry is on the ring.
      auto load_group = [&](int gs) {
        wait_free(&s.gempty[gs], (tk_n & 1) ^ 1, 52);
        if (!ok) return;
        if (lane == 0) {
          const int row = (2 * t + gs) * QG * 16;
          ptx::mbar_arrive_expect_tx(&s.gfull[gs], 2u * QG * 2048u);
          ptx::tma_load_2d(s.grp[gs].q, &tq128, 0, row, &s.gfull[gs]);
          ptx::tma_load_2d(s.grp[gs].dO, &tdo128, 0, row, &s.gfull[gs]);
        }
        __syncwarp();
      };
      load_group(0);
      if (nc > 0 && ok) {   // the token's pooled-key tile, into coarse slot tk_n % 2
        const int cs = (int)(tk_n & 1);
        wait_free(&s.cempty[cs], ((tk_n >> 1) & 1) ^ 1, 52);
        if (ok && lane == 0) {
          ptx::mbar_arrive_expect_tx(&s.cfull[cs], (uint32_t)sizeof(CoarseTile));
          ptx::bulk_load(&s.crs[cs].t, ctile + (size_t)t * sizeof(CoarseTile), (uint32_t)sizeof(CoarseTile),
                         &s.cfull[cs]);
        }
        __syncwarp();
      }
      for (int gs = 0; gs < 2 && ok; ++gs) {
        const int gi = 2 * t + gs;
        const int64_t bh = (int64_t)gi * QG / n1;
        const int c = cnt[gs] < 0 ? 0 : (cnt[gs] > QG * K1 ? QG * K1 : cnt[gs]);
        const int32_t* ul = ulist + (int64_t)gi * QG * K1;
        const int nchunks = (c + CK - 1) / CK;
        for (int ci = 0; ci < nchunks && ok; ++ci) {
          const int ix = ci * CK + (lane & 7);
          const int w0 = __shfl_sync(0xffffffffu, e0[gs], ix & 31);
          const int w1 = __shfl_sync(0xffffffffu, e1[gs], ix & 31);
          int e = ix < 32 ? w0 : w1;
          if (ix >= 64 && ix < c) e = ul[ix];        // unions longer than 64 (K_1 > 8)
          const int nq = c - ci * CK < CK ? c - ci * CK : CK;
          emit(kChunk, gi, gs, bh, nq, ci == 0 ? kFirst : 0, e >> 8, e & 0xff);
          if (gs == 0 && ci == 0 && ok) load_group(1);
        }
        if (ok) emit(kTail, gi, gs, bh, 0, nchunks == 0 ? kFirst : 0, 0, 0);
        if (gs == 0 && nchunks == 0 && ok) load_group(1);
      }
    }
    if (ok) announce(tk_n, -1);
    if (ok) {   // the end marker: the MMA and softmax warps leave their loops on it
      const int slot = (int)(issued % NSLOT);
      wait_free(&s.empty[slot], ((issued / NSLOT) & 1) ^ 1, 53);
      if (ok && lane == 0) {
        s.meta[slot].kind = kEnd;
        ptx::mbar_arrive(&s.full[slot]);
      }
      __syncwarp();
      if (ok) ++issued;
    }
    // do not leave while copies this warp issued may still be landing
    if (lane == 0) {
      for (uint32_t i = issued > NSLOT ? issued - NSLOT : 0; i < issued; ++i)
        ptx::mbar_wait_bounded(&s.full[i % NSLOT], (i / NSLOT) & 1, kWaitLimitNs);
      if (tk_n > 0)
        for (int gs = 0; gs < 2; ++gs) ptx::mbar_wait_bounded(&s.gfull[gs], (tk_n - 1) & 1, kWaitLimitNs);
      if (nc > 0)   // the last two tokens' pooled-key tiles
        for (uint32_t k = tk_n > 2 ? tk_n - 2 : 0; k < tk_n; ++k)
          ptx::mbar_wait_bounded(&s.cfull[k & 1], (k >> 1) & 1, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ============================================================ MMA issue
    // Converged warp, one elected lane issues.  Descriptors are built once and
    // advanced by adding to their start-address field (16-byte units, no
    // carry: shared addresses are below 256 KB).
    constexpr uint32_t idS = tc::idesc_bf16(128, 128, 0, 0);   // S, dP: A = Q / dO (K-major), B = K / V (K-major)
    constexpr uint32_t idSc = tc::idesc_bf16(128, 32, 0, 0);   // the same against the 32 pooled keys
    constexpr uint32_t idQ = tc::idesc_bf16(128, 64, 0, 1);    // dQ += dS K: A = dS (K-major), B = K (MN-major)
    constexpr uint32_t idG = tc::idesc_bf16(64, 64, 1, 1);     // pooled gradients: A = dS_c / P_c (MN), B = Q / dO (MN)
    constexpr uint64_t kSlotStep = sizeof(ChunkSlot) >> 4, kGrpStep = sizeof(GroupSlot) >> 4,
                       kCrsStep = sizeof(CoarseSlot) >> 4;
    const uint64_t dk0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].k), 16, 1024);
    const uint64_t dv0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].v), 16, 1024);
    const uint64_t dq0 = tc::sw128_desc(ptx::smem_u32(s.grp[0].q), 16, 1024);
    const uint64_t do0 = tc::sw128_desc(ptx::smem_u32(s.grp[0].dO), 16, 1024);
    const uint64_t dck0 = tc::sw128_desc(ptx::smem_u32(s.crs[0].t.k), 16, 1024);
    const uint64_t dcv0 = tc::sw128_desc(ptx::smem_u32(s.crs[0].t.v), 16, 1024);
    const uint64_t dsA = tc::sw128_desc(ptx::smem_u32(s.sbuf), 16, 1024);        // dS as a K-major A operand
    const uint64_t dsB = tc::sw128_desc(ptx::smem_u32(s.sbuf), 16384, 1024);     // dS_c / P_c as MN-major operands
    bool ok = true;
    // S side (one entry ahead)
    uint32_t seen = 0, sch = 0, tk_s = 0;
    struct Entry { int kind, slot, gs, nq, flags; uint32_t tk; };
    auto next_s = [&](Entry& c) -> bool {
      const int slot = (int)(seen % NSLOT);
      if (!ptx::mbar_wait_bounded(&s.full[slot], (seen / NSLOT) & 1, kWaitLimitNs)) {
        ok = false;
        return false;
      }
      const Meta& m = s.meta[slot];
      if (m.kind == kEnd) return false;
      c.kind = m.kind;
      c.slot = slot;
      c.gs = m.gs;
      c.nq = m.nq;
      c.flags = m.flags;
      c.tk = tk_s;
      ++seen;
      if (c.flags & kFirst) {   // the group's Q and dO have landed
        if (!ptx::mbar_wait_bounded(&s.gfull[c.gs], tk_s & 1, kWaitLimitNs)) {
          ok = false;
          return false;
        }
      }
      const bool has_s = c.kind == kChunk ? c.nq > 0 : nc > 0;
      if (c.kind == kTail && nc > 0 && c.gs == 0) {   // the token's pooled-key tiles are built
        if (!ptx::mbar_wait_bounded(&s.cfull[tk_s & 1], (tk_s >> 1) & 1, kWaitLimitNs)) {
          ok = false;
          return false;
        }
      }
      if (c.kind == kTail && c.gs == 1) ++tk_s;
      if (has_s) {
        // the softmax warps have read S / dP of the previous entry
        if (!ptx::mbar_wait_bounded(&s.s_empty, (sch & 1) ^ 1, kWaitLimitNs)) {
          ok = false;
          return false;
        }
        tc::fence_after_sync();
        const uint64_t go = kGrpStep * (uint64_t)c.gs;
        if (c.kind == kChunk) {
          const uint64_t so = kSlotStep * (uint64_t)slot;
          if (tc::elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {   // K steps of 16 channels: 32 bytes inside the 128-byte rows
              tc::mma_bf16(tbase + COL_S, dq0 + go + 2u * k, dk0 + so + 2u * k, idS, k > 0);
              tc::mma_bf16(tbase + COL_DP, do0 + go + 2u * k, dv0 + so + 2u * k, idS, k > 0);
            }
            tc::commit(&s.s_full);
          }
        } else {
          const uint64_t co = kCrsStep * (uint64_t)(c.tk & 1);
          if (tc::elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              tc::mma_bf16(tbase + COL_S, dq0 + go + 2u * k, dck0 + co + 2u * k, idSc, k > 0);
              tc::mma_bf16(tbase + COL_DP, do0 + go + 2u * k, dcv0 + co + 2u * k, idSc, k > 0);
            }
            tc::commit(&s.s_full);
          }
        }
        __syncwarp();
        ++sch;
      }
      return true;
    };

    // dQ side
    uint32_t pch = 0;
    bool dq_started = false;
    auto finish = [&](const Entry& c) {
      const uint64_t go = kGrpStep * (uint64_t)c.gs;
      const uint32_t dqc = tbase + COL_DQ;
      const bool has_s = c.kind == kChunk ? c.nq > 0 : nc > 0;
      if (has_s) {
        if (!ptx::mbar_wait_bounded(&s.p_full, pch & 1, kWaitLimitNs)) {
          ok = false;
          return;
        }
        if (!dq_started) {   // the group's first dQ MMA overwrites the accumulator: wait until the last group's was read
          if (!ptx::mbar_wait_bounded(&s.acc_empty, (uint32_t)(c.gs ^ 1), kWaitLimitNs)) {
            ok = false;
            return;
          }
        }
        if (c.kind == kTail && c.gs == 0) {   // the token's first pooled-gradient MMA: the sums were read
          if (!ptx::mbar_wait_bounded(&s.cacc_empty, (c.tk & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
            return;
          }
        }
        tc::fence_after_sync();
        if (c.kind == kChunk) {
          const uint64_t so = kSlotStep * (uint64_t)c.slot;
          if (tc::elect_one()) {
#pragma unroll
            for (int k = 0; k < 8; ++k)     // 16 keys per K step: A 8 TMEM columns, B 2 KB
              tc::mma_bf16_ta(dqc, tbase + COL_DS + 8u * k, dk0 + so + 128u * k, idQ, dq_started || k > 0);
            tc::commit(&s.p_empty);
            tc::commit(&s.empty[c.slot]);
          }
        } else {
          const uint64_t co = kCrsStep * (uint64_t)(c.tk & 1);
          if (tc::elect_one()) {
#pragma unroll
            for (int k = 0; k < 2; ++k)     // dQ += dS_c Kc: 32 pooled keys
              tc::mma_bf16(dqc, dsA + 2u * k, dck0 + co + 128u * k, idQ, dq_started || k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k) {   // dS_c^T Q, P_c^T dO over the group's 128 queries: [pooled key][channel]
              const bool acc = c.gs == 1 || k > 0;   // the token's second group adds to the first's sums
              tc::mma_bf16(tbase + COL_GK, dsB + 128u * k, dq0 + go + 128u * k, idG, acc);
              tc::mma_bf16(tbase + COL_GV, dsB + 1024u + 128u * k, do0 + go + 128u * k, idG, acc);
            }
            tc::commit(&s.p_empty);
          }
        }
        __syncwarp();
        dq_started = true;
        ++pch;
      }
      if (c.kind == kTail) {
        if (!dq_started) {   // no dQ MMA in this group: still hand the (unused) accumulator over in order
          if (!ptx::mbar_wait_bounded(&s.acc_empty, (uint32_t)(c.gs ^ 1), kWaitLimitNs)) {
            ok = false;
            return;
          }
        }
        if (tc::elect_one()) {
          if (!has_s) ptx::mbar_arrive(&s.empty[c.slot]);   // nothing of this entry in flight
          else tc::commit(&s.empty[c.slot]);
          tc::commit(&s.acc_full);           // the group's dQ is complete
          tc::commit(&s.gempty[c.gs]);       // its Q and dO are free
          if (c.gs == 1 && nc > 0) {
            tc::commit(&s.cacc_full);        // the token's pooled-key gradients are complete
            tc::commit(&s.cempty[c.tk & 1]);
          }
        }
        __syncwarp();
        dq_started = false;
      } else if (!has_s) {
        if (tc::elect_one()) ptx::mbar_arrive(&s.empty[c.slot]);
        __syncwarp();
      }
    };

    Entry cur;
    bool have = next_s(cur);
    while (have && ok) {
      Entry nxt;
      const bool have_next = next_s(nxt);
      if (!ok) break;
      finish(cur);
      cur = nxt;
      have = have_next;
    }
    if (!ok && lane == 0) report(err, 54);
    // every MMA issued here has finished before TMEM is released
    if (tc::elect_one()) tc::commit(&s.drain);
    __syncwarp();
    ptx::mbar_wait_bounded(&s.drain, 0, kWaitLimitNs);
  } else if (warp < SOFT_WARPS) {
    // ============================================================ softmax
    const int sub = warp & 3, part = warp >> 2;         // TMEM subpartition; key blocks 2 part, 2 part + 1
    const int row = sub * 32 + lane;                    // query row of the group
    const int qbl = row >> 4;                           // its query block within the group
    const float log2B = log2f((float)g.B);
    const float sc2 = g.scale * kLog2e;
    const bool enrich1 = g.emask & 1u;
    const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
    const int r7 = row & 7;
    const uint32_t rrow = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);   // the row inside a 16 KB half
    uint32_t i = 0, ch = 0, tk = 0;
    // LSE (log2 domain) and D of this thread's row in the current group,
    // loaded at the group's first entry (their latency hides behind the wait
    // for its first S)
    float l2 = 0.f, Dq = 0.f;
    // 16 keys of the row (16-byte chunks 2 j, 2 j + 1 of the row in a 16 KB half); values, not a pointer,
    // so that the words stay in registers
    auto store_row16 = [&](unsigned char* half, int j, uint4 w0, uint4 w1) {
      *reinterpret_cast<uint4*>(half + rrow + ((uint32_t)((2 * j) ^ r7) << 4)) = w0;
      *reinterpret_cast<uint4*>(half + rrow + ((uint32_t)((2 * j + 1) ^ r7) << 4)) = w1;
    };
    while (true) {
      const int slot = (int)(i % NSLOT);
      if (!ptx::mbar_wait_bounded(&s.full[slot], (i / NSLOT) & 1, kWaitLimitNs)) {
        report(err, 55);
        break;
      }
      const Meta& m = s.meta[slot];
      if (m.kind == kEnd) break;
      const int kind = m.kind, gs = m.gs, nq = m.nq, flags = m.flags, gi = m.gi;
      unsigned mine = 0;
      if (kind == kChunk) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int kbi = 2 * part + t;
          if (kbi < nq) mine |= (((unsigned)m.msk[kbi] >> qbl) & 1u) << t;
        }
      }
      // only the meta words are needed from the slot (the MMA warp releases the tiles): release it now
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.empty[slot]);
      if (flags & kFirst) {
        const int64_t grow = (int64_t)gi * QG * 16 + row;
        l2 = lse[grow] * kLog2e;
        Dq = Dws[grow];
      }
      const bool has_s = kind == kChunk ? nq > 0 : nc > 0;
      if (has_s) {
        if (!ptx::mbar_wait_bounded(&s.s_full, ch & 1, kWaitLimitNs)) {
          report(err, 57);
          break;
        }
        tc::fence_after_sync();
        if (kind == kChunk) {
          const unsigned need = __reduce_or_sync(0xffffffffu, mine);   // blocks some row of this warp needs
          uint32_t dw[2][8];
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            uint32_t sr[16], pr[16];
            if ((need >> t) & 1u) {
              const uint32_t col = (uint32_t)((2 * part + t) * 16);
              tc::tmem_ld16(tl + COL_S + col, sr);
              tc::tmem_ld16(tl + COL_DP + col, pr);
              tc::tmem_wait_ld();
            }
            if (t == 1) {   // both blocks read: the MMA warp may overwrite S / dP
              tc::fence_before_sync();
              __syncwarp();
              if (lane == 0) ptx::mbar_arrive(&s.s_empty);
            }
            if ((mine >> t) & 1u) {
              float dsc = 0.f;
              if (enrich1) {   // the block's pooled level-1 token: mean logit + ln B, mean dP
                float zs = 0.f, dps = 0.f;
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                  zs += __uint_as_float(sr[n]);
                  dps += __uint_as_float(pr[n]);
                }
                const float pc = ptx::ex2(fmaf(zs * (1.f / 16.f), sc2, log2B) - l2);
                dsc = pc * (dps * (1.f / 16.f) - Dq) * (1.f / 16.f);
              }
#pragma unroll
              for (int n = 0; n < 8; ++n) {
                const float p0 = ptx::ex2(fmaf(__uint_as_float(sr[2 * n]), sc2, -l2));
                const float p1 = ptx::ex2(fmaf(__uint_as_float(sr[2 * n + 1]), sc2, -l2));
                dw[t][n] = ptx::pack_bf16(fmaf(p0, __uint_as_float(pr[2 * n]) - Dq, dsc),
                                          fmaf(p1, __uint_as_float(pr[2 * n + 1]) - Dq, dsc));
              }
            } else {
#pragma unroll
              for (int n = 0; n < 8; ++n) dw[t][n] = 0u;
            }
          }
          // dQ(i - 1) has read the previous dS from TMEM
          if (!ptx::mbar_wait_bounded(&s.p_empty, (ch & 1) ^ 1, kWaitLimitNs)) {
            report(err, 58);
            break;
          }
          tc::fence_after_sync();
#pragma unroll
          for (int t = 0; t < 2; ++t) tc::tmem_st8(tl + COL_DS + 8u * (uint32_t)(2 * part + t), dw[t]);
          tc::tmem_wait_st();
        } else {
          // pooled keys 16 part .. 16 part + 15 (parts 0, 1; parts 2, 3 write the zero padding),
          // 8 at a time
          uint32_t pw[8], dw[8];
          // the tile's bias row came by bulk copy: observe its barrier here too
          if (part < 2 && !ptx::mbar_wait_bounded(&s.cfull[tk & 1], (tk >> 1) & 1, kWaitLimitNs)) {
            report(err, 56);
            break;
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t sr[8], pr[8];
            if (part < 2) {
              tc::tmem_ld8(tl + COL_S + 16u * part + 8u * h, sr);
              tc::tmem_ld8(tl + COL_DP + 16u * part + 8u * h, pr);
              tc::tmem_wait_ld();
              const float* bias = s.crs[tk & 1].t.bias + 16 * part + 8 * h;
#pragma unroll
              for (int n = 0; n < 4; ++n) {
                float pv[2], dv2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const float b = bias[2 * n + e];
                  const float p = b == -INFINITY ? 0.f : ptx::ex2(fmaf(__uint_as_float(sr[2 * n + e]), sc2, b) - l2);
                  pv[e] = p;
                  dv2[e] = p * (__uint_as_float(pr[2 * n + e]) - Dq);
                }
                pw[4 * h + n] = ptx::pack_bf16(pv[0], pv[1]);
                dw[4 * h + n] = ptx::pack_bf16(dv2[0], dv2[1]);
              }
            } else {
#pragma unroll
              for (int n = 0; n < 4; ++n) pw[4 * h + n] = dw[4 * h + n] = 0u;
            }
          }
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&s.s_empty);
          if (!ptx::mbar_wait_bounded(&s.p_empty, (ch & 1) ^ 1, kWaitLimitNs)) {
            report(err, 58);
            break;
          }
          // dS_c: half 0, pooled keys 0-63; P_c: half 1
          store_row16(s.sbuf, part, make_uint4(dw[0], dw[1], dw[2], dw[3]), make_uint4(dw[4], dw[5], dw[6], dw[7]));
          store_row16(s.sbuf + 16384, part, make_uint4(pw[0], pw[1], pw[2], pw[3]), make_uint4(pw[4], pw[5], pw[6], pw[7]));
        }
        ptx::fence_proxy_async();   // the tail's operands are in shared memory
        tc::fence_before_sync();    // a chunk's dS is in TMEM
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&s.p_full);
        ++ch;
      }
      if (kind == kTail && gs == 1) ++tk;
      ++i;
    }
  } else {
    // ============================================================ epilogue
    // Per token: dQ of each group out of TMEM, then the pooled-key gradients.
    const int sub = (warp - EPI_WARP0) & 3;             // == warp % 4, the TMEM subpartition this warp may read
    const int row = sub * 32 + lane;                    // query row of a group
    const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
    bool ok = true;
    auto fail = [&](int code) {
      report(err, code);
      ok = false;
    };
    // dQ = scale * acc of a group
    auto store_dq = [&](int t, uint32_t tk, int gs) {
      // group 2 tk + gs of this CTA: that phase's parity is gs
      if (!ptx::mbar_wait_bounded(&s.acc_full, (uint32_t)gs, kWaitLimitNs)) return fail(61);
      tc::fence_after_sync();
      const int gi = 2 * t + gs;
      const bool any = nc > 0 || ucount[gi] > 0;        // else no MMA wrote the accumulator: dQ = 0
      const int64_t grow = (int64_t)gi * QG * 16 + row;
      uint4* drow = reinterpret_cast<uint4*>(dq + grow * 64);
#pragma unroll
      for (int p4 = 0; p4 < 4; ++p4) {
        uint32_t r16[16];
        tc::tmem_ld16(tl + COL_DQ + 16u * p4, r16);
        tc::tmem_wait_ld();
        uint32_t w[8];
#pragma unroll
        for (int n = 0; n < 8; ++n)
          w[n] = any ? ptx::pack_bf16(__uint_as_float(r16[2 * n]) * g.scale, __uint_as_float(r16[2 * n + 1]) * g.scale)
                     : 0u;
        drow[2 * p4] = make_uint4(w[0], w[1], w[2], w[3]);
        drow[2 * p4 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.acc_empty);
    };
    // The token's pooled-key gradients: pooled key 16 sub + lane (lanes 0-15)
    // holds its 64 channels; one 4-wide fp32 reduction per 4 channels.
    auto coarse_grads = [&](int t, uint32_t tk) {
      if (!ptx::mbar_wait_bounded(&s.cacc_full, tk & 1, kWaitLimitNs)) return fail(62);
      // the tile's ids came by bulk copy: observe its barrier here too
      if (!ptx::mbar_wait_bounded(&s.cfull[tk & 1], (tk >> 1) & 1, kWaitLimitNs)) return fail(62);
      tc::fence_after_sync();
      const CoarseTile& ct = s.crs[tk & 1].t;
      if (16 * sub < nc) {
        const int bh = (2 * t * QG) / n1;
        const int r = 16 * sub + (lane & 15);
        const int tok = r < nc ? ct.tok[r] : -1;
        const int l = ct.level[r];
        const bool mine = lane < 16 && tok >= 0;
        const int64_t off = mine ? g.pyr_off[l] + ((int64_t)bh * g.n[l] + tok) * 64 : 0;
#pragma unroll 1
        for (int p4 = 0; p4 < 4; ++p4) {
          uint32_t gk[16], gv[16];
          tc::tmem_ld16(tl + COL_GK + 16u * p4, gk);
          tc::tmem_ld16(tl + COL_GV + 16u * p4, gv);
          tc::tmem_wait_ld();
          if (mine) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              ptx::red_add_v4(dPK + off + 16 * p4 + 4 * q, __uint_as_float(gk[4 * q]) * g.scale,
                              __uint_as_float(gk[4 * q + 1]) * g.scale, __uint_as_float(gk[4 * q + 2]) * g.scale,
                              __uint_as_float(gk[4 * q + 3]) * g.scale);
              ptx::red_add_v4(dPV + off + 16 * p4 + 4 * q, __uint_as_float(gv[4 * q]), __uint_as_float(gv[4 * q + 1]),
                              __uint_as_float(gv[4 * q + 2]), __uint_as_float(gv[4 * q + 3]));
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&s.cacc_empty);
        ptx::mbar_arrive(&s.cempty[tk & 1]);   // this warp is done with the tile's ids
      }
    };

    for (uint32_t tk = 0; ok; ++tk) {
      const int r = (int)(tk % TRING);
      if (!ptx::mbar_wait_bounded(&s.tid_full[r], (tk / TRING) & 1, kWaitLimitNs)) {
        fail(63);
        break;
      }
      const int t = s.tid[r];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.tid_empty[r]);
      if (t < 0) break;
      store_dq(t, tk, 0);
      if (ok) store_dq(t, tk, 1);
      if (ok && nc > 0) coarse_grads(t, tk);
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

}  // namespace bwdq

// Needs d = 64, B = 16, n_1 a multiple of 16 and at most 32 pooled keys of
// levels >= 2; anything else returns cudaErrorInvalidValue before a launch.
cudaError_t launch_attn_bwd_q_tc(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                 const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                 const int32_t* idx, const int32_t* offs, const int32_t* qlist,
                                 const BwdWorkspace& ws, void* dq, cudaStream_t s) {
  int nc = 0;
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];
  if (g.d != 64 || g.B != 16 || g.n[1] % (2 * bwdq::QG) || g.Kl[1] < 1 || nc > bwdq::COARSE)
    return cudaErrorInvalidValue;
  const int64_t rows = (int64_t)g.BH * g.N;
  CUtensorMap tq128, tdo128;
  RunMaps tk, tv;
  cudaError_t e = make_token_map_box(&tq128, q, rows, bwdq::QG * 16);
  if (e == cudaSuccess) e = make_token_map_box(&tdo128, dO, rows, bwdq::QG * 16);
  if (e == cudaSuccess) e = make_run_maps(&tk, k, rows);
  if (e == cudaSuccess) e = make_run_maps(&tv, v, rows);
  if (e != cudaSuccess) return e;
  const int ngroups = (int)((int64_t)g.BH * g.n[1] / bwdq::QG);
  const int ntokens = ngroups / 2;
  if (ntokens == 0) return cudaSuccess;
  bwdq::q_prep_kernel<<<2 * ntokens, bwdq::PREP_THREADS, 0, s>>>(g, idx, (const __nv_bfloat16*)o,
                                                             (const __nv_bfloat16*)dO, pyrK, pyrV, offs, qlist,
                                                             ws.ulist, ws.ucount, ws.ulist_kv, ws.ucount_kv, ws.D,
                                                             ws.ctile, nc);
  note_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(bwdq::Smem) + 1024;
  e = cudaFuncSetAttribute(bwdq::attn_bwd_q_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = ntokens < sms ? ntokens : sms;
  bwdq::attn_bwd_q_tc_kernel<<<grid, bwdq::THREADS, smem, s>>>(g, tq128, tdo128, tk, tv, lse, ws.D, ws.ulist,
                                                                ws.ucount, ws.ctile, (__nv_bfloat16*)dq, ws.dPK,
                                                                ws.dPV, ws.counter + 1, device_error_word());
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace llsa
