// k_attn_bwd_kv_tc.cu -- key-major pass of the sparse attention backward on
// the 5th-generation tensor cores (tcgen05, accumulators in tensor memory),
// bf16, d = 64, B = 16 (Trainable Log-linear Sparse Attention summary §4.1).
//
// A fine key block (16 keys) takes the query blocks of its level-1 CSC list 8
// at a time: a chunk of 128 queries whose Q and dO tiles TMA stacks into one
// 128-row, 128-byte-swizzled operand each.  Per chunk:
//   S = Qc K^T and dP = dOc V^T             (M = 128 queries, N = 16 keys, K = 64)
//   one thread per query row reads its 16 S and dP values from TMEM and forms
//   P = exp(z - LSE), dS = P (dP - D); the block's pooled level-1 token (mean
//   logit + ln B, mean dP) folds in as P_c / B and dS_c / B on every key
//   (hierarchical KV enrichment, §四), and both go to shared memory as bf16;
//   dV^T += dOc^T P and dK^T += Qc^T dS      (M = 64 channels, N = 16 keys, K = 128)
// with dV^T and dK^T accumulated in TMEM over the block's chunks.  Then the
// pooled-key gradients of levels >= 2 are spread back over the block's
// tokens (divided by B^l) and dK, dV are written.
//
// Warp-specialised pipeline, one CTA per SM:
//   * warp 4, producer: takes key blocks from a global counter (the CSC lists
//     have very uneven lengths), stages each take's lists in shared memory,
//     packs the valid entries into chunks and loads every chunk into one of
//     NSLOT slots with TMA 2-D tile loads of 2 KB blocks, one lane per tile
//     (the per-load issue cost of TMA is the producer's limit);
//   * warp 5, one thread issues every MMA: S and dP of chunk i, then dV and
//     dK of chunk i - 1, so that the tensor core works on chunk i while the
//     softmax warps handle chunk i - 1;
//   * warps 0-3 and 4-7, two softmax groups taking alternate chunks, one
//     thread per query row, each reading its row's LSE and D itself;
//   * warps 8-11, the epilogue of every key block (dV, dK out of TMEM, plus
//     the pooled-key gradients, read when the block's first chunk arrives).
// S / dP and the dV / dK accumulators are double-buffered in TMEM, the P / dS
// operands in shared memory; every hand-off is an mbarrier, every wait is
// bounded, and on a timeout the kernel sets the device error word and stops.
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
constexpr int NSLOT = 5;
constexpr int GROUP = 128;          // threads of one softmax group / of the epilogue warps
constexpr int EPI_WARP0 = 8, PRODUCER_WARP = 12, MMA_WARP = 13;
constexpr int THREADS = 14 * 32;
// arrivals that free a slot: the MMA thread, each softmax warp, each epilogue warp
constexpr int EMPTY_ARRIVALS = 1 + 8 + 4;
constexpr int UNITS = 16;           // key blocks taken from the counter at a time
constexpr int LISTCAP = 512;        // CSC entries of one take staged in shared memory
constexpr int UPL = 4;              // pooled levels (2..5) whose gradients the epilogue keeps in registers
constexpr uint32_t TMEM_COLS = 128;
// S / dP buffer b at columns 32 b (+16 for dP); accumulator buffer a at
// 64 + 32 a (dV; +16 dK)
constexpr uint32_t COL_S = 0, COL_ACC = 64;
constexpr int kLast = 1, kFirst = 2;
enum : int { kEnd = 0, kChunk = 1 };

struct Slot {
  alignas(1024) unsigned char q[CQ * 2048];
  alignas(1024) unsigned char dO[CQ * 2048];
  alignas(1024) unsigned char k[2048];
  unsigned char v[2048];
  int qb[CQ];          // the chunk's query blocks (ids within the slice)
  int meta[4];         // kind, global key block, query blocks in the chunk, flags
};

struct Smem {
  Slot slot[NSLOT];
  alignas(1024) unsigned char pbuf[2][4096];   // P^T operand: [key][query], K-major, two 64-query atoms
  alignas(1024) unsigned char sbuf[2][4096];   // dS^T operand, same layout
  int stage[64];                               // producer: pending query blocks of the next chunk
  int list[LISTCAP];                           // producer: the CSC entries of the key blocks taken
  alignas(8) uint64_t full[NSLOT];             // producer -> chunk landed (1 arrival + bytes)
  uint64_t empty[NSLOT];                       // MMA + every softmax and epilogue warp -> slot free
  uint64_t s_full[2], s_empty[2];              // S / dP in TMEM: MMA -> softmax group b, its 4 warps -> MMA
  uint64_t p_full[2], p_empty[2];              // P / dS operands: softmax group b (4 warps) -> MMA, MMA -> group b
  uint64_t acc_full[2], acc_empty[2];          // accumulators: MMA -> epilogue, epilogue (4 warps) -> MMA
  uint64_t drain;
  uint32_t tmem_base;

};

static_assert(sizeof(Slot) % 1024 == 0 && offsetof(Smem, sbuf) - offsetof(Smem, pbuf) == 8192,
              "operand buffers are addressed with fixed strides");
static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory of one CTA exceeds the 227 KB limit");

// Byte offset of element (key n, query q) of a [16 keys][128 queries] bf16
// operand stored K-major with the 128-byte swizzle: queries 0-63 and 64-127
// are two atoms of 2 KB, keys 0-7 and 8-15 two 8-row groups 1 KB apart.
__device__ __forceinline__ uint32_t kmajor_off(int n, int q) {
  return (uint32_t)((q >> 6) * 2048 + (n >> 3) * 1024 + (n & 7) * 128 + ((((q & 63) >> 3) ^ (n & 7)) << 4) +
                    (q & 7) * 2);
}

__device__ __forceinline__ void report(int* err, int code) {
  if (err) atomicExch(err, code);
}

__global__ void __launch_bounds__(THREADS, 1) attn_bwd_kv_tc_kernel(
    const __grid_constant__ Geo g, const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo, const float* __restrict__ lse,
    const float* __restrict__ Dws, const int32_t* __restrict__ offs, const int32_t* __restrict__ qlist,
    const float* __restrict__ dPK, const float* __restrict__ dPV, __nv_bfloat16* __restrict__ dk,
    __nv_bfloat16* __restrict__ dv, int* counter, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n1 = g.n[1];
  const int64_t slice_entries = (int64_t)n1 * g.Kl[1];
  const int64_t total = (int64_t)g.BH * n1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      ptx::mbar_init(&s.full[i], 1);
      ptx::mbar_init(&s.empty[i], EMPTY_ARRIVALS);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&s.s_full[b], 1);
      ptx::mbar_init(&s.s_empty[b], 4);
      ptx::mbar_init(&s.p_full[b], 4);
      ptx::mbar_init(&s.p_empty[b], 1);
      ptx::mbar_init(&s.acc_full[b], 1);
      ptx::mbar_init(&s.acc_empty[b], 4);
    }
    ptx::mbar_init(&s.drain, 1);
    ptx::fence_mbar_init();
  }
  // Rows of absent query blocks in a partial chunk keep whatever the slot
  // held; start from zeros so that they are always finite.
  {
    uint4* z = reinterpret_cast<uint4*>(&s.slot[0]);
    const int n16 = (int)(sizeof(Slot) * NSLOT / 16);
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
      ptx::prefetch_tmap(&tq);
      ptx::prefetch_tmap(&tdo);
    }
    uint32_t issued = 0;
    bool ok = true;
    // Takes the next slot: waits until both its consumers are done with it.
    auto acquire = [&]() -> int {
      const int slot = (int)(issued % NSLOT);
      const uint32_t use = issued / NSLOT;
      int good = 1;
      if (lane == 0) good = ptx::mbar_wait_bounded(&s.empty[slot], (use & 1) ^ 1, kWaitLimitNs) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) {
        ok = false;
        if (lane == 0) report(err, 31);
      }
      return slot;
    };
    // Emits one chunk of nq query blocks (ids in s.stage[0..nq)) of key block kbg:
    // lane j < nq loads query block j's Q tile, lane 8 + j its dO tile, lanes
    // 16 and 17 the key block's K and V tiles.
    auto emit = [&](int64_t kbg, int64_t bh, int nq, int flags) {
      const int slot = acquire();
      if (!ok) return;
      Slot& sl = s.slot[slot];
      uint64_t* bar = &s.full[slot];
      if (lane < nq) sl.qb[lane] = s.stage[lane];
      __syncwarp();   // the ids are written before lane 0's arrival publishes the slot
      if (lane == 0) {
        sl.meta[0] = kChunk;
        sl.meta[1] = (int)kbg;
        sl.meta[2] = nq;
        sl.meta[3] = flags;
        ptx::fence_proxy_async();
        if (nq > 0)
          ptx::mbar_arrive_expect_tx(bar, 4096u + (uint32_t)nq * 4096u);
        else
          ptx::mbar_arrive(bar);
      }
      __syncwarp();
      if (nq > 0) {
        const int j = lane & 7;
        if (lane < 16 && j < nq) {
          const int row = (int)((bh * n1 + s.stage[j]) * 16);
          if (lane < 8)
            ptx::tma_load_2d(sl.q + j * 2048, &tq, 0, row, bar);
          else
            ptx::tma_load_2d(sl.dO + j * 2048, &tdo, 0, row, bar);
        } else if (lane == 16 || lane == 17) {
          ptx::tma_load_2d(lane == 16 ? sl.k : sl.v, lane == 16 ? &tk : &tv, 0, (int)(kbg * 16), bar);
        }
      }
      __syncwarp();
      ++issued;
    };

    int nxt_l0 = lane == 0 ? atomicAdd(counter, UNITS) : 0;
    while (ok) {
      const int64_t cb = (int64_t)__shfl_sync(0xffffffffu, nxt_l0, 0);
      if (cb >= total) break;
      if (lane == 0) nxt_l0 = atomicAdd(counter, UNITS);   // the take after this one, in flight meanwhile
      const int64_t ce = cb + UNITS < total ? cb + UNITS : total;
      const int64_t bh = cb / n1;
      const int kb0 = (int)(cb - bh * n1);
      // list starts of the taken blocks (lane u holds block cb + u; lane ce - cb the end)
      const int ow = lane <= (int)(ce - cb) ? offs[g.offs_off[1] + bh * (n1 + 1) + kb0 + lane] : 0;
      const int32_t* slist = qlist + g.idx_off[1] + bh * slice_entries;   // this slice's CSC entries
      // The lists of consecutive blocks are consecutive: stage them in one pass.
      const int lo = __shfl_sync(0xffffffffu, ow, 0);
      const int hi = __shfl_sync(0xffffffffu, ow, (int)(ce - cb));
      const bool staged = lo >= 0 && hi >= lo && hi - lo <= LISTCAP && (int64_t)hi <= slice_entries;
      if (staged) {
        for (int e = lane; e < hi - lo; e += 32) s.list[e] = slist[lo + e];
        __syncwarp();
      }
      for (int64_t kbg = cb; kbg < ce && ok; ++kbg) {
        const int ust = __shfl_sync(0xffffffffu, ow, (int)(kbg - cb));
        int len = __shfl_sync(0xffffffffu, ow, (int)(kbg - cb) + 1) - ust;
        if (len < 0 || ust < 0 || ust + (int64_t)len > slice_entries) len = 0;   // never produced by the transpose
        auto entry = [&](int i) -> int { return staged ? s.list[ust - lo + i] : slist[ust + i]; };
        // number of valid entries, so that the last chunk can be flagged
        int nvalid = 0;
        for (int w0 = 0; w0 < len; w0 += 32) {
          const int a = w0 + lane < len ? entry(w0 + lane) : -1;
          nvalid += __popc(__ballot_sync(0xffffffffu, a >= 0 && a < n1));
        }
        const int nchunks = nvalid > 0 ? (nvalid + CQ - 1) / CQ : 1;
        int pending = 0, emitted = 0;
        for (int w0 = 0; w0 < len && ok; w0 += 32) {
          const int a = w0 + lane < len ? entry(w0 + lane) : -1;
          const bool valid = a >= 0 && a < n1;
          const unsigned bal = __ballot_sync(0xffffffffu, valid);
          if (valid) s.stage[pending + __popc(bal & ((1u << lane) - 1u))] = a;
          pending += __popc(bal);
          __syncwarp();
          while (pending >= CQ && ok) {
            ++emitted;
            emit(kbg, bh, CQ, (emitted == nchunks ? kLast : 0) | (emitted == 1 ? kFirst : 0));
            const int rest = pending - CQ;
            const int t = lane < rest ? s.stage[CQ + lane] : 0;
            __syncwarp();
            if (lane < rest) s.stage[lane] = t;
            __syncwarp();
            pending = rest;
          }
        }
        if (ok && (pending > 0 || emitted == 0)) emit(kbg, bh, pending, kLast | (emitted == 0 ? kFirst : 0));
      }
      __syncwarp();
    }
    if (ok) {
      const int slot = acquire();
      if (ok && lane == 0) {
        s.slot[slot].meta[0] = kEnd;
        ptx::mbar_arrive(&s.full[slot]);
      }
      __syncwarp();
      if (ok) ++issued;
    }
    // do not leave while copies this warp issued may still be landing
    if (lane == 0)
      for (uint32_t i = issued > NSLOT ? issued - NSLOT : 0; i < issued; ++i)
        ptx::mbar_wait_bounded(&s.full[i % NSLOT], (i / NSLOT) & 1, kWaitLimitNs);
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ============================================================ MMA issue
    // The whole warp runs this loop converged; one elected lane issues the
    // MMAs and their commits.  Descriptors are built once and advanced by
    // adding to their start-address field (16-byte units, no carry: shared
    // addresses are below 256 KB).
    constexpr uint32_t idS = tc::idesc_bf16(128, 16, 0, 0);
    constexpr uint32_t idG = tc::idesc_bf16(64, 16, 1, 0);
    // slot j's operands sit sizeof(Slot) bytes after slot j - 1's; buffer 1 4 KB after buffer 0
    constexpr uint64_t kSlotStep = sizeof(Slot) >> 4, kBufStep = 4096 >> 4;
    const uint64_t d_q0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].q), 16, 1024);
    const uint64_t d_o0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].dO), 16, 1024);
    const uint64_t d_k0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].k), 16, 1024);
    const uint64_t d_v0 = tc::sw128_desc(ptx::smem_u32(s.slot[0].v), 16, 1024);
    const uint64_t d_p0 = tc::sw128_desc(ptx::smem_u32(s.pbuf[0]), 16, 1024);
    const uint64_t d_s0 = tc::sw128_desc(ptx::smem_u32(s.sbuf[0]), 16, 1024);
    uint32_t i = 0;            // chunk index
    uint32_t sb = 0;           // chunks with queries so far (S / P buffer uses)
    uint32_t acc_use0 = 0, acc_use1 = 0;
    int acc_buf = 0;
    bool in_unit = false;      // the current block has accumulated at least one chunk
    bool ok = true;
    // the previous chunk, whose dV / dK MMAs follow this chunk's S / dP
    bool have_prev = false;
    int p_slot = 0, p_nq = 0, p_flags = 0;
    uint32_t p_sb = 0;

    auto dvdk = [&]() {
      if (p_nq > 0) {
        const int b = (int)(p_sb & 1);
        if (!ptx::mbar_wait_bounded(&s.p_full[b], (p_sb >> 1) & 1, kWaitLimitNs)) {
          ok = false;
          return;
        }
        if (!in_unit) {   // the block's first MMA overwrites an accumulator buffer: wait until it was read
          const uint32_t use = acc_buf ? acc_use1 : acc_use0;
          if (!ptx::mbar_wait_bounded(&s.acc_empty[acc_buf], (use & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
            return;
          }
        }
        tc::fence_after_sync();
        const uint32_t dacc = tbase + COL_ACC + 32u * (uint32_t)acc_buf;
        const uint64_t dob = d_o0 + kSlotStep * (uint64_t)p_slot, dqb = d_q0 + kSlotStep * (uint64_t)p_slot;
        const uint64_t dpb = d_p0 + kBufStep * (uint64_t)b, dsb = d_s0 + kBufStep * (uint64_t)b;
        if (tc::elect_one()) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            // A: 16 queries of the MN-major dO / Q stack (2 KB per k step); B: K-major operand,
            // k step 16 queries = 32 bytes inside a 64-query atom of 2 KB
            const uint64_t boff = (uint64_t)((k >> 2) * 128 + (k & 3) * 2);
            tc::mma_bf16(dacc, dob + 128u * k, dpb + boff, idG, in_unit || k > 0);
            tc::mma_bf16(dacc + 16, dqb + 128u * k, dsb + boff, idG, in_unit || k > 0);
          }
          tc::commit(&s.p_empty[b]);
          tc::commit(&s.empty[p_slot]);
        }
        __syncwarp();
        in_unit = true;
      } else {
        if (tc::elect_one()) ptx::mbar_arrive(&s.empty[p_slot]);
        __syncwarp();
      }
      if (p_flags & kLast) {
        if (in_unit) {
          if (tc::elect_one()) tc::commit(&s.acc_full[acc_buf]);
          __syncwarp();
          if (acc_buf) ++acc_use1; else ++acc_use0;
          acc_buf ^= 1;
        }
        in_unit = false;
      }
    };

    while (ok) {
      const int slot = (int)(i % NSLOT);
      if (!ptx::mbar_wait_bounded(&s.full[slot], (i / NSLOT) & 1, kWaitLimitNs)) {
        ok = false;
        break;
      }
      const Slot& sl = s.slot[slot];
      const int kind = sl.meta[0];
      if (kind == kEnd) break;
      const int nq = sl.meta[2], flags = sl.meta[3];
      if (nq > 0) {
        const int b = (int)(sb & 1);
        if (!ptx::mbar_wait_bounded(&s.s_empty[b], ((sb >> 1) & 1) ^ 1, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t ds = tbase + COL_S + 32u * (uint32_t)b;
        const uint64_t so = kSlotStep * (uint64_t)slot;
        const uint64_t dqb = d_q0 + so, dob = d_o0 + so, dkb = d_k0 + so, dvb = d_v0 + so;
        if (tc::elect_one()) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // K steps of 16 channels = 32 bytes inside the 128-byte rows
            tc::mma_bf16(ds, dqb + 2u * k, dkb + 2u * k, idS, k > 0);
            tc::mma_bf16(ds + 16, dob + 2u * k, dvb + 2u * k, idS, k > 0);
          }
          tc::commit(&s.s_full[b]);
        }
        __syncwarp();
      }
      if (have_prev) {
        dvdk();
        if (!ok) break;
      }
      have_prev = true;
      p_slot = slot;
      p_nq = nq;
      p_flags = flags;
      p_sb = sb;
      if (nq > 0) ++sb;
      ++i;
    }
    if (ok && have_prev) dvdk();
    if (!ok && lane == 0) report(err, 33);
    // every MMA issued here has finished before TMEM is released
    if (tc::elect_one()) tc::commit(&s.drain);
    __syncwarp();
    ptx::mbar_wait_bounded(&s.drain, 0, kWaitLimitNs);
  } else if (warp < EPI_WARP0) {
    // ============================================================ softmax groups
    // Group gsm takes the chunks with queries whose running count is gsm mod 2,
    // with S / dP buffer gsm and operand buffer gsm; every warp still reads the
    // meta words of every chunk and releases every slot.
    const int gsm = warp >> 2;
    const int row = threadIdx.x & (GROUP - 1);     // query row of the chunk
    const float log2B = log2f((float)g.B);
    const float sc2 = g.scale * kLog2e;
    const bool enrich1 = g.emask & 1u;
    const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t tsb = tl + COL_S + 32u * (uint32_t)gsm;
    unsigned char* pbuf = s.pbuf[gsm];
    unsigned char* sbuf = s.sbuf[gsm];
    // byte offsets of this row's 16 key entries in the K-major operand
    const uint32_t obase = (uint32_t)((row >> 6) * 2048 + (row & 7) * 2);
    const int cq = (row & 63) >> 3;
    uint32_t i = 0, sb = 0;

    while (true) {
      const int slot = (int)(i % NSLOT);
      if (!ptx::mbar_wait_bounded(&s.full[slot], (i / NSLOT) & 1, kWaitLimitNs)) {
        report(err, 32);
        break;
      }
      const Slot& sl = s.slot[slot];
      const int kind = sl.meta[0];
      if (kind == kEnd) break;
      const int nq = sl.meta[2];
      if (nq > 0) {
        if ((int)(sb & 1) == gsm) {
          const uint32_t use = sb >> 1;
          // this row's LSE and D, in flight while the S / dP MMAs run
          const bool valid = (row >> 4) < nq;
          float lrow = 0.f, Dq = 0.f;
          if (valid) {
            const int kbg = sl.meta[1];
            const int bh = kbg / n1;
            const int64_t grow = ((int64_t)bh * n1 + sl.qb[row >> 4]) * 16 + (row & 15);
            lrow = lse[grow];
            Dq = Dws[grow];
          }
          if (!ptx::mbar_wait_bounded(&s.s_full[gsm], use & 1, kWaitLimitNs)) {
            report(err, 34);
            break;
          }
          tc::fence_after_sync();
          uint32_t sr[16], pr[16];
          tc::tmem_ld16(tsb, sr);
          tc::tmem_ld16(tsb + 16u, pr);
          tc::tmem_wait_ld();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&s.s_empty[gsm]);
          const float l2 = lrow * kLog2e;
          float p[16], dsv[16];
          float zs = 0.f, dps = 0.f;
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const float z = __uint_as_float(sr[n]);
            const float dp = __uint_as_float(pr[n]);
            zs += z;
            dps += dp;
            p[n] = exp2f(fmaf(z, sc2, -l2));
            dsv[n] = p[n] * (dp - Dq);
          }
          if (enrich1) {
            const float pc = exp2f(fmaf(zs * (1.f / 16.f), sc2, log2B) - l2) * (1.f / 16.f);
            const float dsc = pc * (dps * (1.f / 16.f) - Dq);
#pragma unroll
            for (int n = 0; n < 16; ++n) {
              p[n] += pc;
              dsv[n] += dsc;
            }
          }
          // the operand buffer is free once the MMAs of this group's previous chunk are done
          if (!ptx::mbar_wait_bounded(&s.p_empty[gsm], (use & 1) ^ 1, kWaitLimitNs)) {
            report(err, 35);
            break;
          }
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            const uint32_t o = obase + (uint32_t)((n >> 3) * 1024 + (n & 7) * 128 + ((cq ^ (n & 7)) << 4));
            *reinterpret_cast<__nv_bfloat16*>(pbuf + o) = __float2bfloat16_rn(valid ? p[n] : 0.f);
            *reinterpret_cast<__nv_bfloat16*>(sbuf + o) = __float2bfloat16_rn(valid ? dsv[n] : 0.f);
          }
          ptx::fence_proxy_async();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&s.p_full[gsm]);
        }
        ++sb;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.empty[slot]);   // this warp is done with the slot
      ++i;
    }
  } else {
    // ============================================================ epilogue warps
    const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    const int c = (warp & 3) * 16 + (lane & 15);   // channel held by this lane (TMEM lane 32 w + i <-> row 16 w + i)
    uint32_t i = 0;
    uint32_t acc_use[2] = {0u, 0u};
    int acc_buf = 0;
    bool unit_mma = false;
    float uk = 0.f, uv = 0.f;   // the block's pooled-key gradients on channel c, divided by B^l

    while (true) {
      const int slot = (int)(i % NSLOT);
      if (!ptx::mbar_wait_bounded(&s.full[slot], (i / NSLOT) & 1, kWaitLimitNs)) {
        report(err, 36);
        break;
      }
      const Slot& sl = s.slot[slot];
      const int kind = sl.meta[0];
      if (kind == kEnd) break;
      const int kbg = sl.meta[1];
      const int nq = sl.meta[2];
      const int flags = sl.meta[3];
      if (nq > 0) unit_mma = true;
      if (flags & kFirst) {
        // read now, used at the block's last chunk (the loads overlap the wait for the accumulators)
        const int bh = kbg / n1;
        const int64_t t0 = (int64_t)(kbg - bh * n1) * 16;
        float kk[UPL], vv[UPL], inv[UPL];
#pragma unroll
        for (int j = 0; j < UPL; ++j) {
          const int l = 2 + j;
          kk[j] = vv[j] = inv[j] = 0.f;
          if (l <= g.L && ((g.emask >> (l - 1)) & 1u)) {
            const int64_t off = g.pyr_off[l] + ((int64_t)bh * g.n[l] + t0 / g.Bl[l]) * 64 + c;
            kk[j] = dPK[off];
            vv[j] = dPV[off];
            inv[j] = 1.f / (float)g.Bl[l];
          }
        }
        uk = uv = 0.f;
        for (int l = 2 + UPL; l <= g.L; ++l) {   // deeper hierarchies (rare)
          if (!((g.emask >> (l - 1)) & 1u)) continue;
          const int64_t off = g.pyr_off[l] + ((int64_t)bh * g.n[l] + t0 / g.Bl[l]) * 64 + c;
          uk = fmaf(dPK[off], 1.f / (float)g.Bl[l], uk);
          uv = fmaf(dPV[off], 1.f / (float)g.Bl[l], uv);
        }
#pragma unroll
        for (int j = 0; j < UPL; ++j) {
          uk = fmaf(kk[j], inv[j], uk);
          uv = fmaf(vv[j], inv[j], uv);
        }
      }
      if (flags & kLast) {
        float av[16], ak[16];
        if (unit_mma) {
          const int ab = acc_buf;
          if (!ptx::mbar_wait_bounded(&s.acc_full[ab], acc_use[ab] & 1, kWaitLimitNs)) {
            report(err, 37);
            break;
          }
          tc::fence_after_sync();
          uint32_t vr[16], kr[16];
          const uint32_t ta = tl + COL_ACC + 32u * (uint32_t)ab;
          tc::tmem_ld16(ta, vr);
          tc::tmem_ld16(ta + 16u, kr);
          tc::tmem_wait_ld();
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&s.acc_empty[ab]);
          ++acc_use[ab];
          acc_buf ^= 1;
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            av[n] = __uint_as_float(vr[n]);
            ak[n] = __uint_as_float(kr[n]) * g.scale;
          }
        } else {
#pragma unroll
          for (int n = 0; n < 16; ++n) av[n] = ak[n] = 0.f;
        }
        if (lane < 16) {
          __nv_bfloat16* pk = dk + (int64_t)kbg * 1024 + c;
          __nv_bfloat16* pv = dv + (int64_t)kbg * 1024 + c;
#pragma unroll
          for (int n = 0; n < 16; ++n) {
            pk[n * 64] = __float2bfloat16_rn(ak[n] + uk);
            pv[n * 64] = __float2bfloat16_rn(av[n] + uv);
          }
        }
        unit_mma = false;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s.empty[slot]);   // this warp is done with the slot
      ++i;
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

cudaError_t launch_attn_bwd_kv_tc(const Geo& g, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                                  const CUtensorMap& tdo, const float* lse, const float* D, const int32_t* offs,
                                  const int32_t* qlist, const float* dPK, const float* dPV, void* dk, void* dv,
                                  int* counter, cudaStream_t s) {
  const size_t smem = sizeof(bwdtc::Smem) + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(bwdtc::attn_bwd_kv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  bwdtc::attn_bwd_kv_tc_kernel<<<sms, bwdtc::THREADS, smem, s>>>(
      g, tk, tv, tq, tdo, lse, D, offs, qlist, dPK, dPV, (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, counter,
      device_error_word());
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace llsa
