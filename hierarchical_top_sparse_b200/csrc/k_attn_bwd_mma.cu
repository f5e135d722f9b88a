// k_attn_bwd_mma.cu -- sparse attention backward on the tensor cores (bf16,
// d = 64, B = 16), in two passes (Trainable Log-linear Sparse Attention
// summary §4.1, "trainable" in its title):
//
//  * query-major pass, per query block (16 queries): D = rowsum(dO * O); the
//    logits against the K_1 picked key blocks and the pooled keys of levels
//    >= 2; P = exp(z - LSE), dP = dO V^T, dS = P (dP - D); dQ = scale * dS K.
//    The pooled keys of levels >= 2 are shared by the 16 query blocks under
//    one level-2 token, so a CTA takes one level-2 token at a time, reduces
//    their gradients (scale * dS^T Q and P^T dO) in shared memory and adds
//    them with one fp32 atomic per (pooled token, channel).
//  * key-major pass (k_attn_bwd_kv_tc.cu, on tcgen05), per fine key block,
//    over the query blocks of its level-1 CSC list: dV, dK, and the pooled-key
//    gradients of levels >= 2 spread back over the B^l tokens they average.
//
// A level-1 pooled token is the mean of the 16 keys of the block it stands
// for, and the queries that attend it are exactly those that picked that
// block.  So level-1 enrichment folds into both passes with no extra loads:
// its logit is the mean of the block's 16 fine logits plus ln B, its dP is the
// mean of the 16 fine dP, and its P and dS add P_c / B and dS_c / B to each of
// the block's 16 fine entries (hierarchical KV enrichment, §四).
//
// Every warp streams its own tiles through a small ring of shared-memory
// slots filled by TMA (2-D tile loads of 2 KB blocks with the 128-byte
// swizzle; a 1-D bulk load of the 64-byte LSE row), a few elements ahead of
// the one it computes, so list lengths are unbounded.  Query blocks are
// assigned statically (16 per CTA step, 2 per warp).  Every wait is bounded;
// a warp that gives up sets the device error word, stops computing and,
// before it exits, waits (bounded) for the copies it issued.
#include <math.h>

#include "llsa_internal.cuh"
#include "mma_tiles.cuh"
#include "ptx.cuh"

namespace llsa {
namespace bwdmma {

constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s: a wait this long means something broke
constexpr float kLog2e = 1.4426950408889634f;
constexpr int GB = 16;        // query blocks per query-major CTA step (one level-2 token)
constexpr int COARSE = 32;    // pooled keys of levels >= 2 per query block, at most

// ------------------------------------------------------ per-warp TMA ring

// A warp's ring of R slots of SLOT bytes (1024-aligned), tiles of 2 KB at
// offsets 0, 2048, 4096, the 64-byte rows at EXTRA; meta words describe each
// slot's element (written by the issuing lane before the barrier arrival).
template <int R, int SLOT, int EXTRA>
struct Ring {
  unsigned char* slots;
  uint64_t* full;
  int* meta;
  uint32_t issued;
  uint32_t consumed;

  __device__ __forceinline__ unsigned char* slot(uint32_t i) const { return slots + (i % R) * SLOT; }
  __device__ __forceinline__ uint32_t tile(uint32_t i, int t) const { return ptx::smem_u32(slot(i) + t * 2048); }
  __device__ __forceinline__ const float* extra(uint32_t i) const {
    return reinterpret_cast<const float*>(slot(i) + EXTRA);
  }
  __device__ __forceinline__ int* meta_of(uint32_t i) const { return meta + (i % R) * 4; }
  __device__ __forceinline__ uint64_t* bar(uint32_t i) const { return &full[i % R]; }
  __device__ __forceinline__ bool can_issue() const { return issued < consumed + R; }
  __device__ __forceinline__ bool wait_next() const {
    return ptx::mbar_wait_bounded(&full[consumed % R], (consumed / R) & 1, kWaitLimitNs);
  }
  // After giving up: wait (bounded) for every copy still in flight.
  __device__ __forceinline__ void drain() const {
    for (uint32_t i = consumed; i < issued; ++i) ptx::mbar_wait_bounded(&full[i % R], (i / R) & 1, kWaitLimitNs);
  }
};

__device__ __forceinline__ void report(int* err, int code) {
  if (err) atomicExch(err, code);
}

// ------------------------------------------------------ query-major pass

constexpr int QW = 8;          // warps per CTA
constexpr int QR = 3;          // ring slots per warp
constexpr int QSLOT = 7168;    // header: Q, dO, O tiles + LSE row; entry: K, V tiles
constexpr int QEXTRA = 6144;

struct QSmem {
  alignas(1024) unsigned char ring[QW][QR][QSLOT];
  alignas(1024) unsigned char ck[COARSE * 128];
  alignas(1024) unsigned char cv[COARSE * 128];
  float accK[COARSE * 64];
  float accV[COARSE * 64];
  float cbias[COARSE];
  int crow_l[COARSE];
  int crow_tok[COARSE];
  int meta[QW][QR][4];
  alignas(8) uint64_t full[QW][QR];
};

using QRing = Ring<QR, QSLOT, QEXTRA>;

// Column skew of row r of the pooled-gradient sums (element (r, c) sits at
// column (c + skew(r & 7)) & 63): the 32 lanes of one atomic add of a C tile
// (rows gq, columns 2 tq4 + const) then hit 32 different banks.
__device__ __forceinline__ int acc_skew(int r7) { return 8 * ((r7 >> 1) & 3) + (r7 & 1); }

// Row statistics of one query block for the lane's two C-tile rows (gq, gq + 8).
struct RowStats {
  float lse2[2];   // LSE in the log2 domain
  float D[2];
};

// P and dS of one 16 x 16 logit tile whose rows are the lane's queries.
// `bias` is added to the scaled logit of column c (log2 domain).
__device__ __forceinline__ void softmax_grad_rows(float (*p)[4], float (*ds)[4], const float (*sc)[4],
                                                  const float (*dp)[4], const RowStats& rs, float sc2,
                                                  const float* bias) {
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = e >> 1;
      const float z = fmaf(sc[j][e], sc2, bias ? bias[j * 2 + (e & 1)] : 0.f);
      p[j][e] = exp2f(z - rs.lse2[r]);
      ds[j][e] = p[j][e] * (dp[j][e] - rs.D[r]);
    }
}

__global__ void __launch_bounds__(QW * 32, 1) attn_bwd_q_mma_kernel(
    const __grid_constant__ Geo g, const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
    const __grid_constant__ CUtensorMap to, const __grid_constant__ CUtensorMap tk,
    const __grid_constant__ CUtensorMap tv, const float* __restrict__ lse, const float* __restrict__ pyrK,
    const float* __restrict__ pyrV, const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ dq,
    float* __restrict__ Dws, float* __restrict__ dPK, float* __restrict__ dPV, int* err, int ngroups) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  QSmem& s = *reinterpret_cast<QSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq4 = lane & 3;
  const int K1 = g.Kl[1];
  const float log2B = log2f((float)g.B);
  const float sc2 = g.scale * kLog2e;
  const bool enrich1 = g.emask & 1u;
  int nc = 0;
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];

  if (threadIdx.x == 0) {
    for (int w = 0; w < QW; ++w)
      for (int i = 0; i < QR; ++i) ptx::mbar_init(&s.full[w][i], 1);
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
    s.crow_tok[r] = -1;
  }
  for (int e = threadIdx.x; e < COARSE * 32; e += blockDim.x) {
    reinterpret_cast<uint32_t*>(s.ck)[e] = 0u;
    reinterpret_cast<uint32_t*>(s.cv)[e] = 0u;
  }
  __syncthreads();

  // Groups go to CTAs with a grid stride, so that the CTAs in flight work on
  // neighbouring groups of one (batch, head) slice and share its K/V in L2.
  const int ng_cta = ngroups > (int)blockIdx.x ? (ngroups - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  const int nunits = 2 * ng_cta;
  QRing ring{s.ring[warp][0], s.full[warp], &s.meta[warp][0][0], 0u, 0u};
  if (lane == 0) {
    ptx::prefetch_tmap(&tq);
    ptx::prefetch_tmap(&tdo);
    ptx::prefetch_tmap(&to);
    ptx::prefetch_tmap(&tk);
    ptx::prefetch_tmap(&tv);
  }

  // ---------------------------------------------------------------- producer
  // The warp's elements, in order: for every unit u (query block
  // (blockIdx.x + (u / 2) * gridDim.x) * 16 + 2 * warp + u % 2), a header (its Q, dO, O tiles
  // and LSE row) and then its K_1 picked K/V blocks.
  auto unit_block = [&](int u) -> int64_t {
    return ((int64_t)blockIdx.x + (int64_t)(u >> 1) * gridDim.x) * GB + 2 * warp + (u & 1);
  };
  auto pick_window = [&](int u, int j0) -> int {
    if (u >= nunits) return -1;
    const int j = j0 + lane;
    return j < K1 ? idx[g.idx_off[1] + unit_block(u) * K1 + j] : -1;
  };
  int pu = 0, pj = -1;
  int pw = -1, pw_next = pick_window(0, 0);
  bool live = true;

  auto pump = [&]() {
    while (live && pu < nunits && ring.can_issue()) {
      const int64_t ab = unit_block(pu);
      const uint32_t i = ring.issued;
      unsigned char* sl = ring.slot(i);
      uint64_t* bar = ring.bar(i);
      if (pj < 0) {
        pw = pw_next;
        pw_next = pick_window(pu + 1, 0);
        if (lane == 0) {
          ptx::fence_proxy_async();
          const int row = (int)(ab * 16);
          ptx::mbar_arrive_expect_tx(bar, 3 * 2048 + 64);
          ptx::tma_load_2d(sl, &tq, 0, row, bar);
          ptx::tma_load_2d(sl + 2048, &tdo, 0, row, bar);
          ptx::tma_load_2d(sl + 4096, &to, 0, row, bar);
          ptx::bulk_load(sl + QEXTRA, lse + ab * 16, 64, bar);
        }
      } else {
        if (pj > 0 && (pj & 31) == 0) pw = pick_window(pu, pj);
        const int kb = __shfl_sync(0xffffffffu, pw, pj & 31);
        const bool ok = kb >= 0 && kb < g.n[1];
        if (lane == 0) {
          ring.meta_of(i)[0] = ok ? 1 : 0;
          ptx::fence_proxy_async();
          if (ok) {
            const int64_t bh = ab / g.n[1];
            const int row = (int)((bh * g.n[1] + kb) * 16);
            ptx::mbar_arrive_expect_tx(bar, 4096);
            ptx::tma_load_2d(sl, &tk, 0, row, bar);
            ptx::tma_load_2d(sl + 2048, &tv, 0, row, bar);
          } else {
            ptx::mbar_arrive(bar);   // an index outside its level: an absent key, nothing to load
          }
        }
      }
      __syncwarp();
      ++ring.issued;
      if (++pj == K1) {
        pj = -1;
        ++pu;
      }
    }
  };

  auto wait_next = [&]() -> bool {
    pump();
    if (!live) return false;
    if (!ring.wait_next()) {
      live = false;
      report(err, 21);
      return false;
    }
    return true;
  };

  // ---------------------------------------------------------------- consumer
  for (int gi = blockIdx.x; gi < ngroups; gi += gridDim.x) {
    const int64_t a0g = (int64_t)gi * GB;
    const int64_t bh = a0g / g.n[1];
    const int a0 = (int)(a0g - bh * g.n[1]);
    if (nc > 0) {
      __syncthreads();   // the previous group's sums are flushed
      if (threadIdx.x < nc) {
        const int l = s.crow_l[threadIdx.x];
        int r = threadIdx.x;
        for (int l2 = 2; l2 < l; ++l2)
          if ((g.emask >> (l2 - 1)) & 1u) r -= g.Kl[l2];
        const int64_t grp = a0 / g.Bl[l - 1];
        const int tok = idx[g.idx_off[l] + (bh * g.n[l] + grp) * g.Kl[l] + r];
        s.crow_tok[threadIdx.x] = (tok >= 0 && tok < g.n[l]) ? tok : -1;
      }
      for (int e = threadIdx.x; e < COARSE * 64; e += blockDim.x) {
        s.accK[e] = 0.f;
        s.accV[e] = 0.f;
      }
      __syncthreads();
      for (int item = threadIdx.x; item < nc * 16; item += blockDim.x) {
        const int row = item >> 4, chunk = item & 15;
        const int l = s.crow_l[row], tok = s.crow_tok[row];
        float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
        if (tok >= 0) {
          const int64_t off = g.pyr_off[l] + (bh * g.n[l] + tok) * 64 + chunk * 4;
          kv = *reinterpret_cast<const float4*>(pyrK + off);
          vv = *reinterpret_cast<const float4*>(pyrV + off);
        }
        const uint32_t o2 = ptx::sw128(row, chunk * 4);
        *reinterpret_cast<uint2*>(s.ck + o2) = make_uint2(ptx::pack_bf16(kv.x, kv.y), ptx::pack_bf16(kv.z, kv.w));
        *reinterpret_cast<uint2*>(s.cv + o2) = make_uint2(ptx::pack_bf16(vv.x, vv.y), ptx::pack_bf16(vv.z, vv.w));
      }
      __syncthreads();
    }

    for (int su = 0; su < 2; ++su) {
      const int64_t ab = a0g + 2 * warp + su;
      if (!wait_next()) continue;
      // ------------------------------------------------ header: Q, dO, O, LSE
      const uint32_t hi = ring.consumed;
      const uint32_t qtile = ring.tile(hi, 0), dotile = ring.tile(hi, 1), otile = ring.tile(hi, 2);
      RowStats rs;
      {
        // D = rowsum(dO * O): lane pair (2r, 2r + 1) takes row r, 32 channels each
        const int r = lane >> 1, h = lane & 1;
        float part = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          const int col = h * 32 + c8 * 8;
          const uint4 dov = *reinterpret_cast<const uint4*>(ring.slot(hi) + 2048 + ptx::sw128(r, col));
          const uint4 ov = *reinterpret_cast<const uint4*>(ring.slot(hi) + 4096 + ptx::sw128(r, col));
          const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dov);
          const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 a = __bfloat1622float2(d2[t]), b = __bfloat1622float2(o2[t]);
            part = fmaf(a.x, b.x, part);
            part = fmaf(a.y, b.y, part);
          }
        }
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        if (h == 0) Dws[ab * 16 + r] = part;
        rs.D[0] = __shfl_sync(0xffffffffu, part, gq * 2);
        rs.D[1] = __shfl_sync(0xffffffffu, part, (gq + 8) * 2);
        const float* lrow = ring.extra(hi);
        rs.lse2[0] = lrow[gq] * kLog2e;
        rs.lse2[1] = lrow[gq + 8] * kLog2e;
      }
      (void)otile;
      uint32_t qa[4][4], doa[4][4];
      tiles::load_a(qa, qtile, lane);
      tiles::load_a(doa, dotile, lane);
      float dqa[8][4];
      tiles::zero_acc(dqa);

      // ------------------------------------ pooled keys of levels >= 2
      const uint32_t ckb = ptx::smem_u32(s.ck), cvb = ptx::smem_u32(s.cv);
      for (int k0 = 0; k0 < nc; k0 += 16) {
        float sc[2][4], dp[2][4], p[2][4], ds[2][4];
        tiles::mma_abt(sc, qa, ckb, k0, lane);
        tiles::mma_abt(dp, doa, cvb, k0, lane);
        float bias[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          bias[2 * j] = s.cbias[k0 + j * 8 + 2 * tq4];
          bias[2 * j + 1] = s.cbias[k0 + j * 8 + 2 * tq4 + 1];
        }
        softmax_grad_rows(p, ds, sc, dp, rs, sc2, bias);
        uint32_t dsa[4], pa[4], t[4];
        tiles::pack_a(dsa, ds);
        tiles::pack_a(pa, p);
        tiles::mma_ab(dqa, dsa, ckb, k0, lane);
        // this block's share of the pooled keys' gradients: dS^T Q and P^T dO
        float part[8][4];
        tiles::transpose_a(t, dsa);
        tiles::zero_acc(part);
        tiles::mma_ab(part, t, qtile, 0, lane);
        const bool v0 = k0 + gq < nc, v1 = k0 + gq + 8 < nc;   // padding rows add nothing
        const int sk = acc_skew(gq);
        float* rk0 = s.accK + (k0 + gq) * 64;
        float* rk1 = rk0 + 8 * 64;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = j * 8 + 2 * tq4 + sk;
          if (v0) {
            atomicAdd(rk0 + (c & 63), part[j][0]);
            atomicAdd(rk0 + ((c + 1) & 63), part[j][1]);
          }
          if (v1) {
            atomicAdd(rk1 + (c & 63), part[j][2]);
            atomicAdd(rk1 + ((c + 1) & 63), part[j][3]);
          }
        }
        tiles::transpose_a(t, pa);
        tiles::zero_acc(part);
        tiles::mma_ab(part, t, dotile, 0, lane);
        float* rv0 = s.accV + (k0 + gq) * 64;
        float* rv1 = rv0 + 8 * 64;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = j * 8 + 2 * tq4 + sk;
          if (v0) {
            atomicAdd(rv0 + (c & 63), part[j][0]);
            atomicAdd(rv0 + ((c + 1) & 63), part[j][1]);
          }
          if (v1) {
            atomicAdd(rv1 + (c & 63), part[j][2]);
            atomicAdd(rv1 + ((c + 1) & 63), part[j][3]);
          }
        }
      }
      __syncwarp();
      ++ring.consumed;   // the header slot goes back to the ring

      // ------------------------------------------------ the picked blocks
      for (int j = 0; j < K1; ++j) {
        if (!wait_next()) break;
        const uint32_t ei = ring.consumed;
        if (ring.meta_of(ei)[0]) {
          const uint32_t ktile = ring.tile(ei, 0), vtile = ring.tile(ei, 1);
          float sc[2][4], dp[2][4], p[2][4], ds[2][4];
          tiles::mma_abt(sc, qa, ktile, 0, lane);
          tiles::mma_abt(dp, doa, vtile, 0, lane);
          softmax_grad_rows(p, ds, sc, dp, rs, sc2, nullptr);
          if (enrich1) {
            // the block's pooled level-1 token: mean logit + ln B, mean dP
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const float zs = tiles::quad_sum(sc[0][2 * r] + sc[0][2 * r + 1] + sc[1][2 * r] + sc[1][2 * r + 1]);
              const float dps = tiles::quad_sum(dp[0][2 * r] + dp[0][2 * r + 1] + dp[1][2 * r] + dp[1][2 * r + 1]);
              const float pc = exp2f(fmaf(zs * (1.f / 16.f), sc2, log2B) - rs.lse2[r]);
              const float dsc = pc * (dps * (1.f / 16.f) - rs.D[r]) * (1.f / 16.f);
#pragma unroll
              for (int jj = 0; jj < 2; ++jj) {
                ds[jj][2 * r] += dsc;
                ds[jj][2 * r + 1] += dsc;
              }
            }
          }
          uint32_t dsa[4];
          tiles::pack_a(dsa, ds);
          tiles::mma_ab(dqa, dsa, ktile, 0, lane);
        }
        __syncwarp();
        ++ring.consumed;
      }
      if (!live) continue;

      // ------------------------------------------------ dQ = scale * acc
      const int64_t r0 = ab * 16 + gq;
      __nv_bfloat16* o0 = dq + r0 * 64;
      __nv_bfloat16* o1 = dq + (r0 + 8) * 64;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = j * 8 + 2 * tq4;
        *reinterpret_cast<uint32_t*>(o0 + c) = ptx::pack_bf16(dqa[j][0] * g.scale, dqa[j][1] * g.scale);
        *reinterpret_cast<uint32_t*>(o1 + c) = ptx::pack_bf16(dqa[j][2] * g.scale, dqa[j][3] * g.scale);
      }
    }

    if (nc > 0) {
      __syncthreads();   // every warp's share is in the sums
      for (int e = threadIdx.x; e < nc * 64; e += blockDim.x) {
        const int row = e >> 6, c = e & 63;
        const int tok = s.crow_tok[row];
        if (tok < 0) continue;
        const int l = s.crow_l[row];
        const int64_t off = g.pyr_off[l] + (bh * g.n[l] + tok) * 64 + c;
        const int sidx = row * 64 + ((c + acc_skew(row & 7)) & 63);
        atomicAdd(dPK + off, s.accK[sidx] * g.scale);
        atomicAdd(dPV + off, s.accV[sidx]);
      }
    }
  }
  if (!live) ring.drain();
}

}  // namespace bwdmma

// ------------------------------------------------------------------ launch

bool attn_bwd_mma_supported(const Geo& g) {
  if (!g.bf16 || g.d != 64 || g.B != 16) return false;
  if (g.n[1] % bwdmma::GB) return false;
  if (g.Kl[1] < 1) return false;
  int nc = 0;
  for (int l = 2; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) nc += g.Kl[l];
  if (nc > bwdmma::COARSE) return false;
  if ((int64_t)g.BH * g.N >= (1ll << 31)) return false;
  if ((int64_t)g.BH * g.n[1] * g.Kl[1] >= (1ll << 31)) return false;
  return true;
}

cudaError_t launch_attn_bwd_mma(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                                void* dv, void* workspace, cudaStream_t s) {
  const int64_t rows = (int64_t)g.BH * g.N;
  CUtensorMap tq, tk, tv, to, tdo;
  cudaError_t e = make_token_map(&tq, q, rows);
  if (e == cudaSuccess) e = make_token_map(&tk, k, rows);
  if (e == cudaSuccess) e = make_token_map(&tv, v, rows);
  if (e == cudaSuccess) e = make_token_map(&to, o, rows);
  if (e == cudaSuccess) e = make_token_map(&tdo, dO, rows);
  if (e != cudaSuccess) return e;
  BwdWorkspace ws = carve_bwd_workspace(g, workspace);
  e = cudaMemsetAsync(ws.dPK, 0, ws.zero_bytes, s);   // pooled-key sums and the work counter
  if (e != cudaSuccess) return e;
  const size_t qsmem = sizeof(bwdmma::QSmem) + 1024;
  e = cudaFuncSetAttribute(bwdmma::attn_bwd_q_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qsmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ngroups = (int)((int64_t)g.BH * g.n[1] / bwdmma::GB);
  const int qgrid = ngroups < sms ? ngroups : sms;
  int* err = device_error_word();
  bwdmma::attn_bwd_q_mma_kernel<<<qgrid, bwdmma::QW * 32, qsmem, s>>>(
      g, tq, tdo, to, tk, tv, lse, pyrK, pyrV, idx, (__nv_bfloat16*)dq, ws.D, ws.dPK, ws.dPV, err, ngroups);
  note_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_bwd_kv_tc(g, k, v, tq, tdo, lse, offs, qlist, ws, dk, dv, s);
}

}  // namespace llsa
