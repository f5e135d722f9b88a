// k_attn_bwd_kv_tc.cu -- key-major pass of the sparse attention backward on
// the 5th-generation tensor cores (tcgen05, accumulators in tensor memory),
// bf16, d = 64, B = 16 (Trainable Log-linear Sparse Attention summary §4.1).
//
// Work unit: a key group, 8 consecutive level-1 key blocks (128 keys) of one
// slice.  The query blocks that picked any of them (the union of their 8
// level-1 CSC lists, each with an 8-bit mask of which blocks it picked) are
// taken 8 at a time: a chunk of 128 queries whose Q and dO tiles TMA stacks
// into 128-row, 128-byte-swizzled operands.  Per chunk:
//   S = Qc K_G^T and dP = dOc V_G^T            (M = 128 queries, N = 128 keys, K = 64)
//   one thread per (query row, half of the keys) reads its 64 S and dP values
//   from TMEM and, for each of its 4 key blocks that the row's query block
//   picked, forms P = exp(z - LSE) and dS = P (dP - D), with the block's
//   pooled level-1 token (mean logit + ln B, mean dP) folded in as P_c / B and
//   dS_c / B on every key of the block (hierarchical KV enrichment, §四);
//   blocks it did not pick get zeros;
//   dV += P^T dOc and dK += dS^T Qc            (M = 128 keys, N = 64 channels, K = 128 queries)
// with dV and dK accumulated in TMEM over the group's chunks, in one of two
// accumulator buffers, so that the epilogue of a group overlaps the next
// group's chunks.  The 128 keys of a group lie under one level-2 token, so
// they share every pooled key of levels >= 2: the epilogue adds one pooled
// gradient per channel and level (divided by B^l) and writes dK and dV, one
// key row per thread.
//
// Sharing the union's Q/dO tiles among the group's 8 key blocks moves about
// 2.5x fewer bytes from L2 than gathering them per key block, and N = 128
// tiles run the tensor cores at full rate where N = 16 tiles are bound by the
// cost of issuing each MMA; the price is the masked (query block, key block)
// pairs, computed and discarded.
//
// Warp roles, one CTA per SM (22 warps):
//   * warp 20, producer: claims key groups one at a time from a counter that
//     all CTAs share (the CTAs in flight then work on neighbouring groups and
//     share their Q/dO tiles in L2, and a CTA that drew long unions does not
//     hold up the launch), reads each group's union (prefetched one group
//     ahead), and loads every chunk (one lane
//     per 2 KB tile) into one of NSLOT slots and every group's K and V (one
//     16 KB box each) into one of two key slots, all with TMA;
//   * warp 21, MMA: a converged warp whose elected lane issues the MMAs and
//     commits them to mbarriers;
//   * warps 0-15, softmax: warps w, w + 4, w + 8, w + 12 share TMEM lanes
//     32 (w % 4).. and take key blocks 2 (w / 4) and 2 (w / 4) + 1 of those
//     query rows;
//   * warps 16-19, epilogue: takes the CTA's key groups in claim order from
//     the producer and each group's accumulators when the MMA warp hands them
//     over.
// Every hand-off is an mbarrier, every wait is bounded; on a timeout the
// kernel sets the device error word and stops.
//
// The unions come from the query-major pre-pass (q_prep_kernel): one warp per
// key group merges the group's 8 sorted level-1 CSC lists and writes the
// union in ascending query-block order, each entry (query block << 8) | pick
// mask, into the group's own range of the CSC layout (a union is never longer
// than the lists it merges).
#include <math.h>
#include <stddef.h>

#include "llsa_internal.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {
namespace bwdtc {

constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int CQ = 8;               // query blocks per chunk (128 queries)
constexpr int KG = 8;               // key blocks per group (128 keys)
constexpr int NSLOT = 3;            // chunk slots
constexpr int SOFT_WARPS = 16, PRODUCER_WARP = 20, MMA_WARP = 21, GRAD_WARP = 22;   // warps 16-19: epilogue
constexpr int THREADS = 23 * 32;
constexpr uint32_t TMEM_COLS = 512;
// S 0-127, dP 128-255; accumulator buffer b at 256 + 128 b: dV + 0, dK + 64
constexpr uint32_t COL_S = 0, COL_DP = 128, COL_ACC = 256;
constexpr int kLast = 1, kFirst = 2;
enum : int { kEnd = 0, kChunk = 1 };
// arrivals that free a chunk slot: the MMA thread and each softmax warp
// a chunk slot is freed by both MMA warps (the S / dP warp once it has read the
// meta words, the dV / dK warp once its MMAs are done) and every softmax warp
constexpr int EMPTY_ARRIVALS = 2 + SOFT_WARPS;
constexpr int GRING = 4;            // key-group ids in flight between the producer and the epilogue

struct ChunkSlot {
  alignas(1024) unsigned char q[CQ * 2048];    // [128 queries][64] bf16, 128-byte swizzle
  alignas(1024) unsigned char dO[CQ * 2048];
};

struct KeySlot {
  alignas(1024) unsigned char k[KG * 2048];    // [128 keys][64] bf16, 128-byte swizzle
  alignas(1024) unsigned char v[KG * 2048];
};

struct Meta {
  int kind, kbg0, nq, flags;                   // kbg0: the group's first key block (global)
  int qb[CQ];                                  // the chunk's query blocks (ids within the slice)
  int msk[CQ];                                 // bit j: the query block picked key block kbg0 + j
};

struct Smem {
  ChunkSlot slot[NSLOT];
  KeySlot key[2];
  // P and dS of one chunk as the B operand of dV^T / dK^T: [query][key], keys
  // contiguous (MN-major), 128-byte swizzle; keys 0-63 and 64-127 are two
  // 16 KB halves, each [128 queries][64 keys].
  alignas(1024) unsigned char pbuf[2 * 16384];
  alignas(1024) unsigned char sbuf[2 * 16384];
  Meta meta[NSLOT];
  alignas(8) uint64_t full[NSLOT], empty[NSLOT];
  uint64_t kfull[2], kempty[2];                // key slots: producer -> MMA, MMA -> producer
  uint64_t s_full, s_empty;                    // S / dP in TMEM: MMA -> softmax, softmax (8 warps) -> MMA
  uint64_t p_full, p_empty;                    // P / dS operands: softmax (8 warps) -> MMA, MMA -> softmax
  uint64_t acc_full[2], acc_empty[2];          // accumulator buffers: MMA -> epilogue, epilogue (4 warps) -> MMA
  uint64_t gid_full[GRING], gid_empty[GRING];  // the CTA's key groups in claim order: producer -> epilogue
  uint64_t drain[2];
  int gid[GRING];
  uint32_t tmem_base;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA exceeds the 227 KB limit");
static_assert(sizeof(ChunkSlot) % 1024 == 0 && sizeof(KeySlot) % 1024 == 0,
              "operands are addressed with fixed strides");

__device__ __forceinline__ void report(int* err, int code) {
  if (err) atomicExch(err, code);
}

__global__ void __launch_bounds__(THREADS, 1) attn_bwd_kv_tc_kernel(
    const __grid_constant__ Geo g, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
    const __grid_constant__ RunMaps tq, const __grid_constant__ RunMaps tdo, const float* __restrict__ lse,
    const float* __restrict__ Dws, const int32_t* __restrict__ offs, const int32_t* __restrict__ ulist,
    const int32_t* __restrict__ ucount, const float* __restrict__ dPK, const float* __restrict__ dPV,
    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, int* __restrict__ counter, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n1 = g.n[1];
  const int64_t slice_entries = (int64_t)n1 * g.Kl[1];
  const int ngroups = (int)((int64_t)g.BH * n1 / KG);   // n1 is a multiple of 16: groups never cross slices

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], EMPTY_ARRIVALS);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.kfull[i], 1);
      ptx::mbar_init(&s.kempty[i], 1);
    }
    ptx::mbar_init(&s.s_full, 1);
    ptx::mbar_init(&s.s_empty, SOFT_WARPS);
    ptx::mbar_init(&s.p_full, SOFT_WARPS);
    ptx::mbar_init(&s.p_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s.acc_full[i], 1);
      ptx::mbar_init(&s.acc_empty[i], 4);
    }
    for (int i = 0; i < GRING; ++i) {
      ptx::mbar_init(&s.gid_full[i], 1);
      ptx::mbar_init(&s.gid_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) ptx::mbar_init(&s.drain[i], 1);
    ptx::fence_mbar_init();
  }
  // Rows of absent query blocks in a partial chunk keep whatever the slot
  // held; start from zeros so that they are always finite.
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
      ptx::prefetch_tmap(&tk);
      ptx::prefetch_tmap(&tv);
    }
    if (lane < kRunMax) {
      ptx::prefetch_tmap(&tq.m[lane]);
      ptx::prefetch_tmap(&tdo.m[lane]);
    }
    uint32_t issued = 0, kissued = 0;
    bool ok = true;
    auto wait_free = [&](uint64_t* bar, uint32_t parity, int code) {
      int good = 1;
      if (lane == 0) good = ptx::mbar_wait_bounded(bar, parity, kWaitLimitNs) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) {
        ok = false;
        if (lane == 0) report(err, code);
      }
    };
    // One chunk of nq query blocks of the group at kbg0 (lane j < nq holds
    // member j in pq / pm).  A run of consecutive query blocks is one box of
    // up to four tiles: lane j issues the Q box that starts at member j, lane
    // 8 + j the dO box.
    auto emit = [&](int kbg0, int64_t bh, int nq, int flags, int pq, int pm) {
      const int slot = (int)(issued % NSLOT);
      wait_free(&s.empty[slot], ((issued / NSLOT) & 1) ^ 1, 41);
      if (!ok) return;
      Meta& m = s.meta[slot];
      if (lane < nq) {
        m.qb[lane] = pq;
        m.msk[lane] = pm;
      }

      __syncwarp();
      uint64_t* bar = &s.full[slot];
      if (lane == 0) {
        m.kind = kChunk;
        m.kbg0 = kbg0;
        m.nq = nq;
        m.flags = flags;
        if (nq > 0)
          ptx::mbar_arrive_expect_tx(bar, (uint32_t)nq * 4096u);
        else
          ptx::mbar_arrive(bar);
      }
      __syncwarp();
      const int j = lane & 7;
      const int qj = __shfl_sync(0xffffffffu, pq, j);
      const int box = __shfl_sync(0xffffffffu, run_box(pq, nq, lane), j);
      if (lane < 16 && box > 0) {
        const int row = (int)((bh * n1 + qj) * 16);
        ChunkSlot& cs = s.slot[slot];
        if (lane < 8)
          ptx::tma_load_2d(cs.q + j * 2048, &tq.m[box - 1], 0, row, bar);
        else
          ptx::tma_load_2d(cs.dO + j * 2048, &tdo.m[box - 1], 0, row, bar);
      }
      __syncwarp();
      ++issued;
    };

    // Key groups are claimed one at a time from a counter shared by all
    // CTAs (so that a CTA that drew long unions does not hold up the launch),
    // one group ahead of the one being loaded.  Lane 0 holds the start and
    // size of a group's union; all lanes hold its first 64 entries.
    auto claim = [&]() -> int {
      int v = 0;
      if (lane == 0) v = atomicAdd(counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    auto info = [&](int gi, int& lo, int& cnt) {
      int a = 0, b = 0;
      if (gi < ngroups && lane == 0) {
        const int bh = gi * KG / n1;
        a = offs[g.offs_off[1] + (int64_t)bh * (n1 + 1) + (gi * KG - bh * n1)];
        b = ucount[gi];
      }
      lo = __shfl_sync(0xffffffffu, a, 0);
      cnt = __shfl_sync(0xffffffffu, b, 0);
    };
    auto entries = [&](int gi, int lo, int cnt, int& e0, int& e1) {
      e0 = e1 = 0;
      if (gi < ngroups) {
        const int32_t* ul = ulist + (int64_t)(gi * KG / n1) * slice_entries + lo;
        if (lane < cnt) e0 = ul[lane];
        if (32 + lane < cnt) e1 = ul[32 + lane];
      }
    };
    // hands the group id (or -1: no more) to the epilogue, in claim order
    uint32_t gcount = 0;
    auto announce = [&](int gi) {
      const int r = (int)(gcount % GRING);
      wait_free(&s.gid_empty[r], ((gcount / GRING) & 1) ^ 1, 40);
      if (!ok) return;
      if (lane == 0) {
        s.gid[r] = gi;
        ptx::mbar_arrive(&s.gid_full[r]);
      }
      __syncwarp();
      ++gcount;
    };
    int gi = claim();
    int lo_n = 0, cnt_n = 0, e0n = 0, e1n = 0;
    info(gi, lo_n, cnt_n);
    entries(gi, lo_n, cnt_n, e0n, e1n);
    while (gi < ngroups && ok) {
      const int lo_c = lo_n, cnt_c = cnt_n, e0c = e0n, e1c = e1n;
      const int gnext = claim();     // prefetch the next group's union while this one streams
      info(gnext, lo_n, cnt_n);
      entries(gnext, lo_n, cnt_n, e0n, e1n);
      announce(gi);
      if (!ok) break;

      const int kbg0 = gi * KG;
      const int64_t bh = kbg0 / n1;
      // the group's K and V: one 16 KB box each
      {
        const int ks = (int)(kissued & 1);
        wait_free(&s.kempty[ks], ((kissued >> 1) & 1) ^ 1, 42);
        if (!ok) break;
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&s.kfull[ks], 2u * KG * 2048u);
          ptx::tma_load_2d(s.key[ks].k, &tk, 0, kbg0 * 16, &s.kfull[ks]);
          ptx::tma_load_2d(s.key[ks].v, &tv, 0, kbg0 * 16, &s.kfull[ks]);
        }
        __syncwarp();
        ++kissued;
      }
      const int cnt = cnt_c < 0 ? 0 : cnt_c;
      const int32_t* ul = ulist + bh * slice_entries + lo_c;
      const int nchunks = cnt > 0 ? (cnt + CQ - 1) / CQ : 1;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int idx = c * CQ + (lane & 7);
        const int w0 = __shfl_sync(0xffffffffu, e0c, idx & 31);
        const int w1 = __shfl_sync(0xffffffffu, e1c, idx & 31);
        int e = idx < 32 ? w0 : w1;
        if (idx >= 64 && idx < cnt) e = ul[idx];     // unions longer than 64 (rare)
        const int nq = cnt - c * CQ < CQ ? cnt - c * CQ : CQ;
        const int flags = (c == 0 ? kFirst : 0) | (c == nchunks - 1 ? kLast : 0);
        emit(kbg0, bh, nq > 0 ? nq : 0, flags, e >> 8, e & 0xff);
      }
      gi = gnext;
    }
    if (ok) announce(-1);
    if (ok) {   // the end marker: every consumer leaves its loop on it
      const int slot = (int)(issued % NSLOT);
      wait_free(&s.empty[slot], ((issued / NSLOT) & 1) ^ 1, 43);
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
      for (uint32_t i = kissued > 2 ? kissued - 2 : 0; i < kissued; ++i)
        ptx::mbar_wait_bounded(&s.kfull[i & 1], (i >> 1) & 1, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp == MMA_WARP || warp == GRAD_WARP) {
    // ============================================================ MMA issue
    // Two converged warps, one elected lane each: warp MMA_WARP issues S and
    // dP of every chunk (as soon as the softmax warps have read those of the
    // chunk before), warp GRAD_WARP dV and dK (once the softmax warps have
    // written P and dS), so that neither issue stream waits behind the other.
    // Each reads every chunk's meta words; commits track only the issuing
    // thread's MMAs (S and dP of a chunk have finished before its P / dS
    // exist, so GRAD_WARP's commits cover the chunk and the group).
    // Descriptors are built once and advanced by adding to their
    // start-address field (16-byte units, no carry: shared addresses are
    // below 256 KB).
    constexpr uint32_t idS = tc::idesc_bf16(128, 128, 0, 0);   // S, dP: A = Q / dO (K-major), B = K / V (K-major)
    constexpr uint32_t idG = tc::idesc_bf16(128, 64, 1, 1);    // dV, dK: A = P / dS (MN-major), B = dO / Q (MN-major)
    constexpr uint64_t kSlotStep = sizeof(ChunkSlot) >> 4, kKeyStep = sizeof(KeySlot) >> 4;
    const uint64_t dq0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].q), 16, 1024);
    const uint64_t do0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].dO), 16, 1024);
    const uint64_t dk0 = tc::sw128_desc(ptx::smem_u32(s.key[0].k), 16, 1024);
    const uint64_t dv0 = tc::sw128_desc(ptx::smem_u32(s.key[0].v), 16, 1024);
    const uint64_t dp = tc::sw128_desc(ptx::smem_u32(s.pbuf), 16384, 1024);
    const uint64_t dsd = tc::sw128_desc(ptx::smem_u32(s.sbuf), 16384, 1024);
    const bool is_s = warp == MMA_WARP;
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok && !ptx::mbar_wait_bounded(bar, parity, kWaitLimitNs)) ok = false;
      return ok;
    };
    uint32_t kseen = 0;           // groups started
    uint32_t nch = 0;             // chunks with queries handled
    uint32_t gcount = 0;          // groups closed (GRAD_WARP)
    bool in_group = false;
    for (uint32_t seen = 0; ok; ++seen) {
      const int slot = (int)(seen % NSLOT);
      if (!wait(&s.full[slot], (seen / NSLOT) & 1)) break;
      const Meta& m = s.meta[slot];
      const int kind = m.kind, nq = m.nq, flags = m.flags;
      if (kind == kEnd) break;
      if (flags & kFirst) ++kseen;
      const int ks = (int)((kseen - 1) & 1);
      if (is_s) {
        // the meta words are in registers (the tiles are released by the other warp)
        __syncwarp();
        if (tc::elect_one()) ptx::mbar_arrive(&s.empty[slot]);
        __syncwarp();
        if ((flags & kFirst) && !wait(&s.kfull[ks], ((kseen - 1) >> 1) & 1)) break;
        if (nq == 0) continue;
        // the softmax warps have read S / dP of the previous chunk
        if (!wait(&s.s_empty, (nch & 1) ^ 1)) break;
        tc::fence_after_sync();
        const uint64_t so = kSlotStep * (uint64_t)slot, ko = kKeyStep * (uint64_t)ks;
        if (tc::elect_one()) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // K steps of 16 channels: 32 bytes inside the 128-byte rows
            tc::mma_bf16(tbase + COL_S, dq0 + so + 2u * k, dk0 + ko + 2u * k, idS, k > 0);
            tc::mma_bf16(tbase + COL_DP, do0 + so + 2u * k, dv0 + ko + 2u * k, idS, k > 0);
          }
          tc::commit(&s.s_full);
        }
        __syncwarp();
        ++nch;
        continue;
      }
      // dV / dK of this chunk
      if (nq > 0) {
        if (!wait(&s.p_full, nch & 1)) break;
        const uint32_t b = gcount & 1;
        // the group's first MMA overwrites the buffer: wait until it was read
        if (!in_group && !wait(&s.acc_empty[b], ((gcount >> 1) & 1) ^ 1)) break;
        tc::fence_after_sync();
        const uint64_t so = kSlotStep * (uint64_t)slot;
        const uint32_t acc = tbase + COL_ACC + 128u * b;
        if (tc::elect_one()) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {   // K steps of 16 queries: two 8-row groups = 2 KB
            tc::mma_bf16(acc, dp + 128u * k, do0 + so + 128u * k, idG, in_group || k > 0);
            tc::mma_bf16(acc + 64, dsd + 128u * k, dq0 + so + 128u * k, idG, in_group || k > 0);
          }
          tc::commit(&s.p_empty);
          tc::commit(&s.empty[slot]);
        }
        __syncwarp();
        in_group = true;
        ++nch;
      } else {
        if (tc::elect_one()) ptx::mbar_arrive(&s.empty[slot]);
        __syncwarp();
      }
      if (flags & kLast) {
        const uint32_t b = gcount & 1;
        // no MMA in this group: still hand the buffer over in order
        if (!in_group && !wait(&s.acc_empty[b], ((gcount >> 1) & 1) ^ 1)) break;
        if (tc::elect_one()) {
          tc::commit(&s.kempty[ks]);   // the group's K and V are free once its MMAs are done
          tc::commit(&s.acc_full[b]);
        }
        __syncwarp();
        ++gcount;
        in_group = false;
      }
    }
    if (!ok && lane == 0) report(err, is_s ? 44 : 49);
    // every MMA issued here has finished before TMEM is released
    if (tc::elect_one()) tc::commit(&s.drain[is_s ? 0 : 1]);
    __syncwarp();
    ptx::mbar_wait_bounded(&s.drain[is_s ? 0 : 1], 0, kWaitLimitNs);
  } else if (warp < SOFT_WARPS) {
    // ============================================================ softmax
    const int sub = warp & 3, part = warp >> 2;         // TMEM subpartition; key blocks 2 part, 2 part + 1
    const int row = sub * 32 + lane;                    // query row of the chunk
    const float log2B = log2f((float)g.B);
    const float sc2 = g.scale * kLog2e;
    const bool enrich1 = g.emask & 1u;
    const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
    const int r7 = row & 7;
    // this row's 16-byte chunks of key block kb in the P / dS operands: half kb / 4, chunks 2 (kb % 4) (+1)
    const uint32_t rbase = (uint32_t)((part >> 1) * 16384 + (row >> 3) * 1024 + (row & 7) * 128);
    uint32_t i = 0, ch = 0;
    while (true) {
      const int slot = (int)(i % NSLOT);
      if (!ptx::mbar_wait_bounded(&s.full[slot], (i / NSLOT) & 1, kWaitLimitNs)) {
        report(err, 45);
        break;
      }
      const Meta& m = s.meta[slot];
      if (m.kind == kEnd) break;
      const int nq = m.nq;
      const int blk = row >> 4;
      const bool valid = blk < nq;
      const unsigned mine = valid ? ((unsigned)m.msk[blk] >> (2 * part)) & 3u : 0u;
      const int qbr = valid ? m.qb[blk] : 0;
      const int kbg0 = m.kbg0;
      // only the meta words are needed from the slot (the MMA warp releases the tiles): release it now
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.empty[slot]);
      if (nq > 0) {
        float l2 = 0.f, Dq = 0.f;
        if (mine) {   // this row's LSE and D, in flight while the S / dP MMAs run
          const int bh = kbg0 / n1;
          const int64_t grow = ((int64_t)bh * n1 + qbr) * 16 + (row & 15);
          l2 = lse[grow] * kLog2e;
          Dq = Dws[grow];
        }
        const unsigned need = __reduce_or_sync(0xffffffffu, mine);   // blocks some row of this warp picked
        if (!ptx::mbar_wait_bounded(&s.s_full, ch & 1, kWaitLimitNs)) {
          report(err, 46);
          break;
        }
        tc::fence_after_sync();
        // P and dS of the row's 2 key blocks, packed bf16 pairs; one block's
        // S / dP in registers at a time
        uint32_t pw[2][8], dw[2][8];
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
            float pc = 0.f, dsc = 0.f;
            if (enrich1) {   // the block's pooled level-1 token: mean logit + ln B, mean dP
              float zs = 0.f, dps = 0.f;
#pragma unroll
              for (int n = 0; n < 16; ++n) {
                zs += __uint_as_float(sr[n]);
                dps += __uint_as_float(pr[n]);
              }
              pc = ptx::ex2(fmaf(zs * (1.f / 16.f), sc2, log2B) - l2) * (1.f / 16.f);
              dsc = pc * (dps * (1.f / 16.f) - Dq);
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) {
              const float p0 = ptx::ex2(fmaf(__uint_as_float(sr[2 * n]), sc2, -l2));
              const float p1 = ptx::ex2(fmaf(__uint_as_float(sr[2 * n + 1]), sc2, -l2));
              const float d0 = fmaf(p0, __uint_as_float(pr[2 * n]) - Dq, dsc);
              const float d1 = fmaf(p1, __uint_as_float(pr[2 * n + 1]) - Dq, dsc);
              pw[t][n] = ptx::pack_bf16(p0 + pc, p1 + pc);
              dw[t][n] = ptx::pack_bf16(d0, d1);
            }
          } else {
#pragma unroll
            for (int n = 0; n < 8; ++n) pw[t][n] = dw[t][n] = 0u;
          }
        }
        // the operand buffers are free once the previous chunk's dV / dK MMAs are done
        if (!ptx::mbar_wait_bounded(&s.p_empty, (ch & 1) ^ 1, kWaitLimitNs)) {
          report(err, 46);
          break;
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int j = (2 * part + t) & 3;   // block within its half of the keys
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t o = rbase + ((uint32_t)((2 * j + c) ^ r7) << 4);
            *reinterpret_cast<uint4*>(s.pbuf + o) =
                make_uint4(pw[t][4 * c], pw[t][4 * c + 1], pw[t][4 * c + 2], pw[t][4 * c + 3]);
            *reinterpret_cast<uint4*>(s.sbuf + o) =
                make_uint4(dw[t][4 * c], dw[t][4 * c + 1], dw[t][4 * c + 2], dw[t][4 * c + 3]);
          }
        }
        ptx::fence_proxy_async();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&s.p_full);
        ++ch;
      }
      ++i;
    }
  } else {
    // ============================================================ epilogue
    // Per key group of this CTA (the producer's order): the pooled-key
    // gradients per channel, then dK and dV of key row 32 (warp % 4) + lane
    // out of accumulator buffer k % 2, one 128-byte row each per thread.
    const int sub = warp & 3;
    const int row = sub * 32 + lane;                    // key of the group (TMEM lane)
    const uint32_t tl = tbase + ((uint32_t)(sub * 32) << 16);
    for (uint32_t k = 0;; ++k) {
      const int r = (int)(k % GRING);
      if (!ptx::mbar_wait_bounded(&s.gid_full[r], (k / GRING) & 1, kWaitLimitNs)) {
        report(err, 47);
        break;
      }
      const int gi = s.gid[r];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.gid_empty[r]);
      if (gi < 0) break;
      const int kbg0 = gi * KG;
      const int bh = kbg0 / n1;
      const int64_t t0 = (int64_t)(kbg0 - bh * n1) * 16;   // the group's first key within its slice
      // The group's pooled-key gradients per channel, divided by B^l: lane i
      // holds channels i and 32 + i (each warp computes its own copy, so
      // that no barrier joins the epilogue warps).
      float uk0 = 0.f, uk1 = 0.f, uv0 = 0.f, uv1 = 0.f;
      for (int l = 2; l <= g.L; ++l) {
        if (!((g.emask >> (l - 1)) & 1u)) continue;
        const int64_t off = g.pyr_off[l] + ((int64_t)bh * g.n[l] + t0 / g.Bl[l]) * 64 + lane;
        const float inv = 1.f / (float)g.Bl[l];
        uk0 = fmaf(dPK[off], inv, uk0);
        uk1 = fmaf(dPK[off + 32], inv, uk1);
        uv0 = fmaf(dPV[off], inv, uv0);
        uv1 = fmaf(dPV[off + 32], inv, uv1);
      }
      const uint32_t b = k & 1;
      if (!ptx::mbar_wait_bounded(&s.acc_full[b], (k >> 1) & 1, kWaitLimitNs)) {
        report(err, 48);
        break;
      }
      tc::fence_after_sync();
      const bool any = ucount[gi] > 0;                  // else no MMA wrote the buffer
      const int64_t grow = (int64_t)kbg0 * 16 + row;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {                     // dV, then dK
        uint4* dst = reinterpret_cast<uint4*>((h == 0 ? dv : dk) + grow * 64);
        const float u0 = h == 0 ? uv0 : uk0, u1 = h == 0 ? uv1 : uk1;
        const float f = h == 0 ? 1.f : g.scale;
#pragma unroll
        for (int p4 = 0; p4 < 4; ++p4) {
          uint32_t r16[16];
          tc::tmem_ld16(tl + COL_ACC + 128u * b + 64u * (uint32_t)h + 16u * p4, r16);
          tc::tmem_wait_ld();
          uint32_t w[8];
#pragma unroll
          for (int n = 0; n < 8; ++n) {
            const int c = 16 * p4 + 2 * n;                // channel of the pair
            const float b0 = __shfl_sync(0xffffffffu, c < 32 ? u0 : u1, c & 31);
            const float b1 = __shfl_sync(0xffffffffu, c + 1 < 32 ? u0 : u1, (c + 1) & 31);
            const float a0 = any ? __uint_as_float(r16[2 * n]) * f : 0.f;
            const float a1 = any ? __uint_as_float(r16[2 * n + 1]) * f : 0.f;
            w[n] = ptx::pack_bf16(a0 + b0, a1 + b1);
          }
          dst[2 * p4] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[2 * p4 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.acc_empty[b]);
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

}  // namespace bwdtc

// Needs n_1 to be a multiple of 16 (checked by the caller): key groups of 8
// blocks never cross a slice and lie under one level-2 token.
cudaError_t launch_attn_bwd_kv_tc(const Geo& g, const void* k, const void* v, const RunMaps& tq,
                                  const RunMaps& tdo, const float* lse, const int32_t* offs,
                                  const BwdWorkspace& ws, void* dk, void* dv, cudaStream_t s) {
  CUtensorMap tk, tv;   // one box = one key group (8 blocks, 128 rows)
  cudaError_t e = make_token_map_box(&tk, k, (int64_t)g.BH * g.N, bwdtc::KG * 16);
  if (e == cudaSuccess) e = make_token_map_box(&tv, v, (int64_t)g.BH * g.N, bwdtc::KG * 16);
  if (e != cudaSuccess) return e;
  const int ngroups = (int)((int64_t)g.BH * g.n[1] / bwdtc::KG);
  const size_t smem = sizeof(bwdtc::Smem) + 1024;
  e = cudaFuncSetAttribute(bwdtc::attn_bwd_kv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = ngroups < sms ? ngroups : sms;
  bwdtc::attn_bwd_kv_tc_kernel<<<grid, bwdtc::THREADS, smem, s>>>(g, tk, tv, tq, tdo, lse, ws.D, offs, ws.ulist_kv,
                                                                   ws.ucount_kv, ws.dPK, ws.dPV, (__nv_bfloat16*)dk,
                                                                   (__nv_bfloat16*)dv, ws.counter, device_error_word());
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace llsa
