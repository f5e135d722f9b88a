// k_transpose.cu -- sparse index transpose (query-major lists -> key-major lists).
//
// Follows the CSR -> CSC transpose of the popular write-up of arXiv:2512.16615
// (§四) and of the Trainable Log-linear Sparse Attention summary (§4.1): count
// per key how many queries picked it, exclusive prefix sum of the counts as
// offsets, scatter every query id into its key's range.  Every launch covers
// all levels at once.  Counting and scattering use warp-aggregated atomics:
// lanes holding the same key elect one leader that adds the group's size.
// The scatter order is arbitrary, so a last pass writes each key's ids in
// ascending order (short ranges by an in-register rank, long ranges through a
// shared-memory bitmap of the query ids).
#include "llsa_internal.cuh"

namespace llsa {

__device__ __forceinline__ int level_of(const int64_t* off, int L, int64_t e) {
  int l = 1;
  while (l < L && e >= off[l + 1]) ++l;
  return l;
}

// Adds `active` lanes' ones to base[key] with one atomic per distinct key in the
// warp; returns this lane's slot (old value + rank inside its key group).
// Every lane of the warp must call it.
__device__ __forceinline__ int warp_aggregated_reserve(int* base, long long key, bool active) {
  const int lane = threadIdx.x & 31;
  const unsigned grp = __match_any_sync(0xffffffffu, active ? key : -1ll);
  const int leader = __ffs(grp) - 1;
  int old = 0;
  if (active && lane == leader) old = atomicAdd(base + key, __popc(grp));
  old = __shfl_sync(0xffffffffu, old, leader);
  return old + __popc(grp & ((1u << lane) - 1u));
}

struct TransposeArgs {
  const int32_t* idx;
  int32_t* offs;
  int32_t* qlist;
  int32_t* cursor;   // [sum_l BH * n_l]: counts, then fill positions
  int32_t* tmp;      // unsorted query lists, same layout as qlist
};

__global__ void count_kernel(Geo g, TransposeArgs a) {
  const int64_t total = g.idx_off[g.L + 1];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) & ~31ll; base < total; base += stride) {
    const int64_t e = base + (threadIdx.x & 31);
    bool active = e < total;
    long long key = 0;
    if (active) {
      const int l = level_of(g.idx_off, g.L, e);
      const int64_t le = e - g.idx_off[l];
      const int64_t per = (int64_t)g.n[l] * g.Kl[l];
      const int64_t bh = le / per;
      const int32_t j = a.idx[e];
      if (j < 0 || j >= g.n[l]) active = false;   // never produced by the selection
      key = g.cur_off[l] + bh * g.n[l] + j;
    }
    warp_aggregated_reserve(a.cursor, key, active);
  }
}

// One block per (level, slice): exclusive scan of the counts into offs; the
// cursors restart at each key's offset for the scatter.
__global__ void __launch_bounds__(1024) scan_kernel(Geo g, TransposeArgs a) {
  __shared__ int wsum[32];
  __shared__ int carry_s;
  const int l = 1 + blockIdx.x / g.BH;
  const int bh = blockIdx.x % g.BH;
  const int n = g.n[l];
  int32_t* cnt = a.cursor + g.cur_off[l] + (int64_t)bh * n;
  int32_t* offs = a.offs + g.offs_off[l] + (int64_t)bh * (n + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int j = base + threadIdx.x;
    const int v = j < n ? cnt[j] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
      int wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      wsum[lane] = wi - w;                 // exclusive prefix of the warp sums
    }
    __syncthreads();
    const int carry = carry_s;
    const int excl = carry + wsum[warp] + incl - v;
    if (j < n) {
      offs[j] = excl;
      cnt[j] = excl;
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry_s = excl + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) offs[n] = carry_s;
}

__global__ void scatter_kernel(Geo g, TransposeArgs a) {
  const int64_t total = g.idx_off[g.L + 1];
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) & ~31ll; base < total; base += stride) {
    const int64_t e = base + (threadIdx.x & 31);
    bool active = e < total;
    long long key = 0;
    int64_t list_base = 0;
    int q = 0;
    if (active) {
      const int l = level_of(g.idx_off, g.L, e);
      const int64_t le = e - g.idx_off[l];
      const int64_t per = (int64_t)g.n[l] * g.Kl[l];
      const int64_t bh = le / per;
      q = (int)((le - bh * per) / g.Kl[l]);
      const int32_t j = a.idx[e];
      if (j < 0 || j >= g.n[l]) active = false;   // never produced by the selection
      key = g.cur_off[l] + bh * g.n[l] + j;
      list_base = g.idx_off[l] + bh * per;
    }
    const int slot = warp_aggregated_reserve(a.cursor, key, active);
    if (active) a.tmp[list_base + slot] = q;
  }
}

constexpr int kSortWarps = 8;
constexpr int kBitmapWords = 256;    // 8192 query ids per window (a small array keeps 8 blocks per SM resident)

// One warp per (level, slice, key): writes the key's query ids ascending.
__global__ void __launch_bounds__(kSortWarps * 32) sort_kernel(Geo g, TransposeArgs a) {
  __shared__ unsigned bitmap[kSortWarps][kBitmapWords];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t key = (int64_t)blockIdx.x * kSortWarps + warp;
  if (key >= g.cur_off[g.L + 1]) return;
  const int l = level_of(g.cur_off, g.L, key);
  const int64_t lk = key - g.cur_off[l];
  const int n = g.n[l];
  const int64_t bh = lk / n;
  const int j = (int)(lk - bh * n);
  const int32_t* offs = a.offs + g.offs_off[l] + bh * (n + 1);
  const int start = offs[j], len = offs[j + 1] - start;
  if (len <= 0) return;
  const int64_t list_base = g.idx_off[l] + bh * (int64_t)n * g.Kl[l] + start;
  const int32_t* src = a.tmp + list_base;
  int32_t* dst = a.qlist + list_base;
  if (len <= 32) {
    const int v = lane < len ? src[lane] : 0x7fffffff;
    int rank = 0;
    for (int i = 0; i < 32; ++i) rank += __shfl_sync(0xffffffffu, v, i) < v;
    if (lane < len) dst[rank] = v;
    return;
  }
  unsigned* bm = bitmap[warp];
  int written = 0;
  for (int win = 0; win < n; win += kBitmapWords * 32) {
    const int span = min(kBitmapWords * 32, n - win);
    const int words = (span + 31) >> 5;
    for (int w = lane; w < words; w += 32) bm[w] = 0u;
    __syncwarp();
    for (int i = lane; i < len; i += 32) {
      const int q = src[i] - win;
      if (q >= 0 && q < span && src[i] < n) atomicOr(&bm[q >> 5], 1u << (q & 31));
    }
    __syncwarp();
    for (int wb = 0; wb < words; wb += 32) {
      const int w = wb + lane;
      unsigned bits = w < words ? bm[w] : 0u;
      const int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = written + incl - c;
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        dst[pos++] = win + w * 32 + b;
      }
      written += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
  }
}

cudaError_t launch_index_transpose(const Geo& g, const int32_t* idx, int32_t* offs, int32_t* qlist,
                                   int32_t* scratch, cudaStream_t s) {
  TransposeArgs a;
  a.idx = idx;
  a.offs = offs;
  a.qlist = qlist;
  a.cursor = scratch;
  size_t cur_bytes = ((size_t)g.cur_off[g.L + 1] * sizeof(int32_t) + 255) & ~(size_t)255;
  a.tmp = (int32_t*)((char*)scratch + cur_bytes);
  cudaError_t e = cudaMemsetAsync(a.cursor, 0, (size_t)g.cur_off[g.L + 1] * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  const int64_t entries = g.idx_off[g.L + 1];
  int64_t blocks = (entries + 255) / 256;
  int grid = (int)(blocks < 148 * 8 ? (blocks > 0 ? blocks : 1) : 148 * 8);
  count_kernel<<<grid, 256, 0, s>>>(g, a);
  scan_kernel<<<g.L * g.BH, 1024, 0, s>>>(g, a);
  scatter_kernel<<<grid, 256, 0, s>>>(g, a);
  const int64_t keys = g.cur_off[g.L + 1];
  sort_kernel<<<(int)((keys + kSortWarps - 1) / kSortWarps), kSortWarps * 32, 0, s>>>(g, a);
  note_launches(4);
  return cudaGetLastError();
}

}  // namespace llsa

// ----------------------------------------------- transpose without scratch
//
// llsa_index_transpose_noalloc: the same four kernels, with their scratch in a
// fixed device array owned by this library instead of a caller buffer.  The
// array is a file-scope __device__ object, so every GPU that loads the library
// holds kNoAllocScratchBytes of it until the process exits.  Host code cannot
// use the symbol's name as a device address: every call looks up its address
// on the current device with cudaGetSymbolAddress (a host-side lookup, no
// launch), so that a device reset between calls cannot leave a stale address.

namespace llsa {

constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.
static llsa_status noalloc_scratch(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return LLSA_ERR_CUDA;
  *out = ptr;
  return LLSA_OK;
}

}  // namespace llsa

extern "C" llsa_status llsa_index_transpose_noalloc(const llsa_problem* p, const int32_t* idx, int32_t* offs,
                                                    int32_t* qlist, llsa_stream stream) {
  llsa::Geo g;
  llsa_status st = llsa::make_geo(p, &g);
  if (st != LLSA_OK) return st;
  const void* bufs[3] = {idx, offs, qlist};
  for (const void* b : bufs) {
    if (!b) return LLSA_ERR_ARG;
    if ((uintptr_t)b & 15u) return LLSA_ERR_ALIGN;
  }
  const size_t cur = ((size_t)g.cur_off[g.L + 1] * sizeof(int32_t) + 255) & ~(size_t)255;
  const size_t need = cur + (size_t)g.idx_off[g.L + 1] * sizeof(int32_t);
  if (need > llsa::kNoAllocScratchBytes) return LLSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = llsa::noalloc_scratch(&scratch);
  if (st != LLSA_OK) return st;
  cudaError_t e = llsa::launch_index_transpose(g, idx, offs, qlist, (int32_t*)scratch, (cudaStream_t)stream);
  if (e != cudaSuccess || cudaPeekAtLastError() != cudaSuccess) return LLSA_ERR_CUDA;
  return LLSA_OK;
}
