// k_attn_simt.cu -- sparse attention forward and backward on the CUDA cores
// (fp32 FMA), the path for fp32 problems.
//
// One 128-thread block per query block of B fine queries.  All B queries of a
// block share one key set (hierarchical KV enrichment, Trainable Log-linear
// Sparse Attention summary §四): the B tokens of every level-1 block in
// S_1(a), then, for each enriched level l, the pooled tokens S_l(floor(a /
// B^(l-1))) with logit bias ln(B^l).  Keys stream through shared memory in
// chunks of 32; the softmax is the usual running max / running sum.
// Backward (§4.1): a query-major pass computes dQ and the pooled-key
// gradients; a key-major pass walks the level-1 key-major (CSC) lists to build
// dK and dV of every fine key block without atomics and adds the pooled
// gradients back to the B^l tokens each pooled token averages.
#include <math.h>

#include "llsa_internal.cuh"

namespace llsa {

constexpr int kThreads = 128;
constexpr int kChunk = 32;
constexpr int kDMax = 128;

template <typename T>
__device__ __forceinline__ const T* tok_row(const T* base, const Geo& g, int bh, int64_t tok) {
  return base + ((int64_t)bh * g.N + tok) * g.d;
}

// Number of keys of one query block and the description of key m.
struct KeySet {
  int nfine;          // K_1 * B fine keys
  int total;          // fine + pooled keys
};

__device__ __forceinline__ KeySet key_set_size(const Geo& g) {
  KeySet ks;
  ks.nfine = g.Kl[1] * g.B;
  ks.total = ks.nfine;
  for (int l = 1; l <= g.L; ++l)
    if ((g.emask >> (l - 1)) & 1u) ks.total += g.Kl[l];
  return ks;
}

// Resolves key m of query block a: level 0 (fine token id) or level l >= 1
// (pooled token id).  Returns the level; writes the token id.
__device__ __forceinline__ int resolve_key(const Geo& g, const int32_t* idx, int bh, int a, int m, int nfine,
                                           int64_t* tok) {
  // An index outside its level (never produced by the selection kernels) makes
  // the key absent instead of reading outside the tensors.
  if (m < nfine) {
    const int32_t* s1 = idx + g.idx_off[1] + ((int64_t)bh * g.n[1] + a) * g.Kl[1];
    const int32_t blk = s1[m / g.B];
    *tok = (int64_t)blk * g.B + m % g.B;
    return (blk >= 0 && blk < g.n[1]) ? 0 : -1;
  }
  m -= nfine;
  for (int l = 1; l <= g.L; ++l) {
    if (!((g.emask >> (l - 1)) & 1u)) continue;
    if (m < g.Kl[l]) {
      const int64_t grp = a / g.Bl[l - 1];
      const int32_t* sl = idx + g.idx_off[l] + ((int64_t)bh * g.n[l] + grp) * g.Kl[l];
      *tok = sl[m];
      return (sl[m] >= 0 && sl[m] < g.n[l]) ? l : -1;
    }
    m -= g.Kl[l];
  }
  *tok = 0;
  return -1;
}

// Loads key m's row of K (or V) as fp32 into dst[0..d).
template <typename T>
__device__ __forceinline__ void load_key_elem(const Geo& g, const T* kx, const float* pyr, int bh, int level,
                                              int64_t tok, int c, float* dst) {
  if (level == 0)
    *dst = to_f32(tok_row(kx, g, bh, tok)[c]);
  else
    *dst = pyr[g.pyr_off[level] + ((int64_t)bh * g.n[level] + tok) * g.d + c];
}

struct SimtSmem {
  int d, ldq;          // row stride of Q-like buffers (d + 1)
  int ldp;             // row stride of p / ds (max(kChunk, B) + 1)
  float* q;            // [B][d+1]
  float* g2;           // [B][d+1]  dO (backward)
  float* k;            // [max(kChunk, B)][d+1]
  float* v;            // [max(kChunk, B)][d+1]
  float* p;            // [B][ldp]
  float* ds;           // [B][ldp]
  float* bias;         // [kChunk]
  int* lvl;            // [kChunk]
  int64_t* tok;        // [kChunk]
  float* rowstat;      // [B] lse, [B] D
};

__host__ __device__ inline int simt_rows(int B) { return B > kChunk ? B : kChunk; }

__host__ __device__ inline size_t simt_smem_bytes(int B, int d) {
  const int rk = simt_rows(B);
  size_t f = (size_t)B * (d + 1) * 2 + (size_t)rk * (d + 1) * 2 + (size_t)B * (rk + 1) * 2 + kChunk + 2 * B;
  return f * sizeof(float) + kChunk * (sizeof(int) + sizeof(int64_t)) + 64;
}

__device__ __forceinline__ SimtSmem carve(char* base, int B, int d) {
  SimtSmem s;
  const int rk = simt_rows(B);
  s.d = d;
  s.ldq = d + 1;
  s.ldp = rk + 1;
  float* f = reinterpret_cast<float*>(base);
  s.q = f; f += B * (d + 1);
  s.g2 = f; f += B * (d + 1);
  s.k = f; f += rk * (d + 1);
  s.v = f; f += rk * (d + 1);
  s.p = f; f += B * s.ldp;
  s.ds = f; f += B * s.ldp;
  s.bias = f; f += kChunk;
  s.rowstat = f; f += 2 * B;
  int64_t* t = reinterpret_cast<int64_t*>(((uintptr_t)f + 7) & ~(uintptr_t)7);
  s.tok = t; t += kChunk;
  s.lvl = reinterpret_cast<int*>(t);
  return s;
}

// Fills the chunk's key/value rows (fp32) and biases; keys past the end get
// bias -inf and zero rows.
template <typename T>
__device__ void load_chunk(const Geo& g, SimtSmem& s, const T* k, const T* v, const float* pyrK, const float* pyrV,
                           const int32_t* idx, int bh, int a, int m0, const KeySet& ks) {
  for (int kk = threadIdx.x; kk < kChunk; kk += blockDim.x) {
    const int m = m0 + kk;
    int64_t tok = 0;
    int lvl = -1;
    if (m < ks.total) lvl = resolve_key(g, idx, bh, a, m, ks.nfine, &tok);
    s.tok[kk] = tok;
    s.lvl[kk] = lvl;
    s.bias[kk] = lvl < 0 ? -INFINITY : (lvl == 0 ? 0.f : logf((float)g.Bl[lvl]));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kChunk * g.d; e += blockDim.x) {
    const int kk = e / g.d, c = e - kk * g.d;
    const int lvl = s.lvl[kk];
    float kv = 0.f, vv = 0.f;
    if (lvl >= 0) {
      load_key_elem(g, k, pyrK, bh, lvl, s.tok[kk], c, &kv);
      load_key_elem(g, v, pyrV, bh, lvl, s.tok[kk], c, &vv);
    }
    s.k[kk * s.ldq + c] = kv;
    s.v[kk * s.ldq + c] = vv;
  }
  __syncthreads();
}

// ------------------------------------------------------------------ forward

template <typename T, int B>
__global__ void __launch_bounds__(kThreads) attn_fwd_simt_kernel(Geo g, const T* __restrict__ q,
                                                                 const T* __restrict__ k, const T* __restrict__ v,
                                                                 const float* __restrict__ pyrK,
                                                                 const float* __restrict__ pyrV,
                                                                 const int32_t* __restrict__ idx, T* __restrict__ o,
                                                                 float* __restrict__ lse) {
  constexpr int QT = kThreads / B;           // threads per query
  constexpr int CPT = kDMax / QT;            // channel slots per thread
  constexpr int KPT = kChunk / QT > 0 ? kChunk / QT : 1;
  extern __shared__ __align__(16) char smem_raw[];
  SimtSmem s = carve(smem_raw, B, g.d);
  const int bh = blockIdx.x / g.n[1];
  const int a = blockIdx.x % g.n[1];
  const int qi = threadIdx.x / QT, sub = threadIdx.x % QT;
  const int d = g.d;
  const KeySet ks = key_set_size(g);

  for (int e = threadIdx.x; e < B * d; e += blockDim.x) {
    const int r = e / d, c = e - r * d;
    s.q[r * s.ldq + c] = to_f32(tok_row(q, g, bh, (int64_t)a * B + r)[c]);
  }
  float acc[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) acc[j] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  for (int m0 = 0; m0 < ks.total; m0 += kChunk) {
    __syncthreads();
    load_chunk(g, s, k, v, pyrK, pyrV, idx, bh, a, m0, ks);
    float z[KPT];
    float cmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < KPT; ++jj) {
      const int kk = sub + jj * QT;
      float sc = -INFINITY;
      if (kk < kChunk) {
        float dot = 0.f;
        for (int c = 0; c < d; ++c) dot = fmaf(s.q[qi * s.ldq + c], s.k[kk * s.ldq + c], dot);
        sc = s.bias[kk] == -INFINITY ? -INFINITY : fmaf(dot, g.scale, s.bias[kk]);
      }
      z[jj] = sc;
      cmax = fmaxf(cmax, sc);
    }
#pragma unroll
    for (int o2 = QT / 2; o2 > 0; o2 >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o2));
    const float m_new = fmaxf(m_run, cmax);
    const float alpha = m_run == -INFINITY ? 0.f : expf(m_run - m_new);
    float psum = 0.f;
#pragma unroll
    for (int jj = 0; jj < KPT; ++jj) {
      const int kk = sub + jj * QT;
      const float pv = z[jj] == -INFINITY ? 0.f : expf(z[jj] - m_new);
      if (kk < kChunk) s.p[qi * s.ldp + kk] = pv;
      psum += pv;
    }
#pragma unroll
    for (int o2 = QT / 2; o2 > 0; o2 >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o2);
    l_run = l_run * alpha + psum;
    m_run = m_new;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = sub + j * QT;
      if (c < d) {
        float t = acc[j] * alpha;
        for (int kk = 0; kk < kChunk; ++kk) t = fmaf(s.p[qi * s.ldp + kk], s.v[kk * s.ldq + c], t);
        acc[j] = t;
      }
    }
  }
  const float inv = 1.f / l_run;
  T* orow = o + ((int64_t)bh * g.N + (int64_t)a * B + qi) * d;
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = sub + j * QT;
    if (c < d) orow[c] = from_f32<T>(acc[j] * inv);
  }
  if (sub == 0) lse[(int64_t)bh * g.N + (int64_t)a * B + qi] = m_run + logf(l_run);
}

// ----------------------------------------------- backward, query-major pass

// dQ for every query and the pooled-key gradients (atomically summed over the
// blocks that attend each pooled token).  Also writes D_i = dO_i . o_i.
template <typename T, int B>
__global__ void __launch_bounds__(kThreads) attn_bwd_q_simt_kernel(
    Geo g, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ o,
    const T* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ pyrK,
    const float* __restrict__ pyrV, const int32_t* __restrict__ idx, T* __restrict__ dq, float* __restrict__ Dws,
    float* __restrict__ dPK, float* __restrict__ dPV) {
  constexpr int QT = kThreads / B;
  constexpr int CPT = kDMax / QT;
  constexpr int KPT = kChunk / QT > 0 ? kChunk / QT : 1;
  extern __shared__ __align__(16) char smem_raw[];
  SimtSmem s = carve(smem_raw, B, g.d);
  const int bh = blockIdx.x / g.n[1];
  const int a = blockIdx.x % g.n[1];
  const int qi = threadIdx.x / QT, sub = threadIdx.x % QT;
  const int d = g.d;
  const KeySet ks = key_set_size(g);
  const int64_t row0 = (int64_t)bh * g.N + (int64_t)a * B;

  for (int e = threadIdx.x; e < B * d; e += blockDim.x) {
    const int r = e / d, c = e - r * d;
    s.q[r * s.ldq + c] = to_f32(q[(row0 + r) * d + c]);
    s.g2[r * s.ldq + c] = to_f32(dO[(row0 + r) * d + c]);
  }
  __syncthreads();
  {
    float part = 0.f;
    for (int c = sub; c < d; c += QT) part = fmaf(s.g2[qi * s.ldq + c], to_f32(o[(row0 + qi) * d + c]), part);
#pragma unroll
    for (int o2 = QT / 2; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
    if (sub == 0) {
      s.rowstat[qi] = lse[row0 + qi];
      s.rowstat[B + qi] = part;
      Dws[row0 + qi] = part;
    }
  }
  float acc[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) acc[j] = 0.f;

  for (int m0 = 0; m0 < ks.total; m0 += kChunk) {
    __syncthreads();
    load_chunk(g, s, k, v, pyrK, pyrV, idx, bh, a, m0, ks);
    const float lse_q = s.rowstat[qi], D_q = s.rowstat[B + qi];
#pragma unroll
    for (int jj = 0; jj < KPT; ++jj) {
      const int kk = sub + jj * QT;
      if (kk >= kChunk) continue;
      float pv = 0.f, dsv = 0.f;
      if (s.bias[kk] != -INFINITY) {
        float dot = 0.f, dpd = 0.f;
        for (int c = 0; c < d; ++c) {
          dot = fmaf(s.q[qi * s.ldq + c], s.k[kk * s.ldq + c], dot);
          dpd = fmaf(s.g2[qi * s.ldq + c], s.v[kk * s.ldq + c], dpd);
        }
        pv = expf(fmaf(dot, g.scale, s.bias[kk]) - lse_q);
        dsv = pv * (dpd - D_q);
      }
      s.p[qi * s.ldp + kk] = pv;
      s.ds[qi * s.ldp + kk] = dsv;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = sub + j * QT;
      if (c < d) {
        float t = acc[j];
        for (int kk = 0; kk < kChunk; ++kk) t = fmaf(s.ds[qi * s.ldp + kk], s.k[kk * s.ldq + c], t);
        acc[j] = t;
      }
    }
    // pooled keys of this chunk: reduce over the block's B queries, one atomic per (token, channel)
    for (int e = threadIdx.x; e < kChunk * d; e += blockDim.x) {
      const int kk = e / d, c = e - kk * d;
      const int lvl = s.lvl[kk];
      if (lvl < 1) continue;
      float gk = 0.f, gv = 0.f;
      for (int r = 0; r < B; ++r) {
        gk = fmaf(s.ds[r * s.ldp + kk], s.q[r * s.ldq + c], gk);
        gv = fmaf(s.p[r * s.ldp + kk], s.g2[r * s.ldq + c], gv);
      }
      const int64_t off = g.pyr_off[lvl] + ((int64_t)bh * g.n[lvl] + s.tok[kk]) * d + c;
      atomicAdd(dPK + off, gk * g.scale);
      atomicAdd(dPV + off, gv);
    }
  }
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = sub + j * QT;
    if (c < d) dq[(row0 + qi) * d + c] = from_f32<T>(acc[j] * g.scale);
  }
}

// ------------------------------------------------- backward, key-major pass

// One block per fine key block: gathers the query blocks that picked it from
// the level-1 CSC lists, accumulates dK and dV in registers, then adds the
// pooled-key gradients of every enriched level divided by B^l.
template <typename T, int B>
__global__ void __launch_bounds__(kThreads) attn_bwd_kv_simt_kernel(
    Geo g, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ dO,
    const float* __restrict__ lse, const int32_t* __restrict__ offs, const int32_t* __restrict__ qlist,
    const float* __restrict__ Dws, const float* __restrict__ dPK, const float* __restrict__ dPV,
    T* __restrict__ dk, T* __restrict__ dv) {
  constexpr int QT = kThreads / B;
  constexpr int CPT = kDMax / QT;
  extern __shared__ __align__(16) char smem_raw[];
  SimtSmem s = carve(smem_raw, B, g.d);   // q, g2: gathered query block; k, v: this key block (first B rows)
  const int bh = blockIdx.x / g.n[1];
  const int kb = blockIdx.x % g.n[1];
  const int d = g.d;
  const int kj = threadIdx.x / QT, sub = threadIdx.x % QT;   // key row owned for accumulation
  const int64_t krow0 = (int64_t)bh * g.N + (int64_t)kb * B;
  for (int e = threadIdx.x; e < B * d; e += blockDim.x) {
    const int r = e / d, c = e - r * d;
    s.k[r * s.ldq + c] = to_f32(k[(krow0 + r) * d + c]);
    s.v[r * s.ldq + c] = to_f32(v[(krow0 + r) * d + c]);
  }
  float ak[CPT], av[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) ak[j] = av[j] = 0.f;
  const int32_t* of = offs + g.offs_off[1] + (int64_t)bh * (g.n[1] + 1);
  const int32_t* ql = qlist + g.idx_off[1] + (int64_t)bh * g.n[1] * g.Kl[1];
  const int beg = of[kb], end = of[kb + 1];
  for (int it = beg; it < end; ++it) {
    const int a = ql[it];
    if (a < 0 || a >= g.n[1]) continue;       // never produced by the transpose
    const int64_t qrow0 = (int64_t)bh * g.N + (int64_t)a * B;
    __syncthreads();
    for (int e = threadIdx.x; e < B * d; e += blockDim.x) {
      const int r = e / d, c = e - r * d;
      s.q[r * s.ldq + c] = to_f32(q[(qrow0 + r) * d + c]);
      s.g2[r * s.ldq + c] = to_f32(dO[(qrow0 + r) * d + c]);
    }
    for (int r = threadIdx.x; r < B; r += blockDim.x) {
      s.rowstat[r] = lse[qrow0 + r];
      s.rowstat[B + r] = Dws[qrow0 + r];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < B * B; e += blockDim.x) {
      const int r = e / B, c2 = e - r * B;      // query r, key c2
      float dot = 0.f, dpd = 0.f;
      for (int c = 0; c < d; ++c) {
        dot = fmaf(s.q[r * s.ldq + c], s.k[c2 * s.ldq + c], dot);
        dpd = fmaf(s.g2[r * s.ldq + c], s.v[c2 * s.ldq + c], dpd);
      }
      const float pv = expf(dot * g.scale - s.rowstat[r]);
      s.p[r * s.ldp + c2] = pv;
      s.ds[r * s.ldp + c2] = pv * (dpd - s.rowstat[B + r]);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = sub + j * QT;
      if (c < d) {
        float tk = ak[j], tv = av[j];
        for (int r = 0; r < B; ++r) {
          tk = fmaf(s.ds[r * s.ldp + kj], s.q[r * s.ldq + c], tk);
          tv = fmaf(s.p[r * s.ldp + kj], s.g2[r * s.ldq + c], tv);
        }
        ak[j] = tk;
        av[j] = tv;
      }
    }
  }
  const int64_t t = (int64_t)kb * B + kj;      // fine token id of the owned row
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    const int c = sub + j * QT;
    if (c >= d) continue;
    float gk = ak[j] * g.scale, gv = av[j];
    for (int l = 1; l <= g.L; ++l) {
      if (!((g.emask >> (l - 1)) & 1u)) continue;
      const int64_t off = g.pyr_off[l] + ((int64_t)bh * g.n[l] + t / g.Bl[l]) * d + c;
      const float inv = 1.f / (float)g.Bl[l];
      gk = fmaf(dPK[off], inv, gk);
      gv = fmaf(dPV[off], inv, gv);
    }
    dk[(krow0 + kj) * d + c] = from_f32<T>(gk);
    dv[(krow0 + kj) * d + c] = from_f32<T>(gv);
  }
}

// ------------------------------------------------------------------ launch

template <typename T, int B>
static cudaError_t fwd_simt(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                            const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s) {
  const size_t smem = simt_smem_bytes(B, g.d);
  auto kern = attn_fwd_simt_kernel<T, B>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kern<<<g.BH * g.n[1], kThreads, smem, s>>>(g, (const T*)q, (const T*)k, (const T*)v, pyrK, pyrV, idx, (T*)o, lse);
  note_launches(1);
  return cudaGetLastError();
}

template <typename T, int B>
static cudaError_t bwd_simt(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                            const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                            const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                            void* dv, float* Dws, float* dPK, float* dPV, cudaStream_t s) {
  const size_t smem = simt_smem_bytes(B, g.d);
  auto kq = attn_bwd_q_simt_kernel<T, B>;
  auto kkv = attn_bwd_kv_simt_kernel<T, B>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kq<<<g.BH * g.n[1], kThreads, smem, s>>>(g, (const T*)q, (const T*)k, (const T*)v, (const T*)o, (const T*)dO, lse,
                                           pyrK, pyrV, idx, (T*)dq, Dws, dPK, dPV);
  note_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kkv<<<g.BH * g.n[1], kThreads, smem, s>>>(g, (const T*)q, (const T*)k, (const T*)v, (const T*)dO, lse, offs, qlist,
                                            Dws, dPK, dPV, (T*)dk, (T*)dv);
  note_launches(1);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t fwd_simt_any(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                                const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s) {
  switch (g.B) {
    case 4: return fwd_simt<T, 4>(g, q, k, v, pyrK, pyrV, idx, o, lse, s);
    case 16: return fwd_simt<T, 16>(g, q, k, v, pyrK, pyrV, idx, o, lse, s);
    case 64: return fwd_simt<T, 64>(g, q, k, v, pyrK, pyrV, idx, o, lse, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_fwd_simt(const Geo& g, const void* q, const void* k, const void* v, const float* pyrK,
                                 const float* pyrV, const int32_t* idx, void* o, float* lse, cudaStream_t s) {
  if (g.bf16) return fwd_simt_any<__nv_bfloat16>(g, q, k, v, pyrK, pyrV, idx, o, lse, s);
  return fwd_simt_any<float>(g, q, k, v, pyrK, pyrV, idx, o, lse, s);
}

template <typename T>
static cudaError_t bwd_simt_any(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                                void* dv, float* Dws, float* dPK, float* dPV, cudaStream_t s) {
  switch (g.B) {
    case 4: return bwd_simt<T, 4>(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, Dws, dPK, dPV, s);
    case 16: return bwd_simt<T, 16>(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, Dws, dPK, dPV, s);
    case 64: return bwd_simt<T, 64>(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, Dws, dPK, dPV, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_bwd_simt(const Geo& g, const void* q, const void* k, const void* v, const void* o,
                                 const void* dO, const float* lse, const float* pyrK, const float* pyrV,
                                 const int32_t* idx, const int32_t* offs, const int32_t* qlist, void* dq, void* dk,
                                 void* dv, void* workspace, cudaStream_t s) {
  const BwdWorkspace ws = carve_bwd_workspace(g, workspace);
  float* Dws = ws.D;
  float* dPK = ws.dPK;
  float* dPV = ws.dPV;
  cudaError_t e = cudaMemsetAsync(dPK, 0, 2 * bwd_pyr_bytes(g), s);
  if (e != cudaSuccess) return e;
  if (g.bf16)
    return bwd_simt_any<__nv_bfloat16>(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, Dws, dPK,
                                       dPV, s);
  return bwd_simt_any<float>(g, q, k, v, o, dO, lse, pyrK, pyrV, idx, offs, qlist, dq, dk, dv, Dws, dPK, dPV, s);
}

}  // namespace llsa
