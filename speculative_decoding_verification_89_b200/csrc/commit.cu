// Paged-KV commit / rollback and pruning of the buffered rows.
//
// HiSpec (gist.science summary of arXiv 2510.01336), section 2: KV entries
// and hidden states are buffered while drafting and the entries of rejected
// tokens are dropped before the next phase ("Wiederverwendung von KV-Cache und
// versteckten Zustaenden"); paged attention with block tables lets every
// sequence accept its own number of tokens without padding ("Unterstuetzung
// fuer Batch-Inferenz").
//
// Two launches. (1) One CTA plans: it checks every sequence, the pool and the
// stack before anything changes, then frees table tails (sequences ascending,
// tails in ascending index, pushed) and allocates missing blocks (sequences
// ascending, popped), sets the lengths and the packed hidden-row offsets. The
// allocation order couples all sequences, hence the single CTA. (2) Many CTAs
// copy each kept token's staged K/V rows into its pool slot and its hidden
// row into the packed output (16-byte vectors, streaming hints).
#include "common.cuh"
#include "kernels.cuh"

namespace specv {

constexpr int kPlanThreads = 1024;
constexpr int kCopyThreads = 256;
constexpr int kCopyParts = 4;  // CTAs per kept token

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Block-wide exclusive scan of one int per thread (kPlanThreads threads).
__device__ int block_excl_scan(int v, int* total) {
  __shared__ int warp_sums[kPlanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_sums[lane] = wi - w;  // exclusive
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - v;
  // Total: last thread's inclusive value.
  __shared__ int s_total;
  if (threadIdx.x == blockDim.x - 1) s_total = excl + v;
  __syncthreads();
  *total = s_total;
  __syncthreads();  // warp_sums / s_total reusable afterwards
  return excl;
}

__global__ void __launch_bounds__(kPlanThreads) commit_plan_kernel(CommitArgs a) {
  grid_dependency_wait();
  extern __shared__ int s_nb[];  // [B] blocks covered before the commit
  __shared__ int s_bad, s_code;
  if (threadIdx.x == 0) { s_bad = 0; s_code = 0; }
  __syncthreads();
  if (a.status && *(volatile int32_t*)a.status != SPEC_OK) return;  // sticky error
  const int bs = a.block_size;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) s_nb[b] = ceil_div(max(a.seq_lens[b], 0), bs);
  __syncthreads();
  // Every covered table entry must be a valid block id: one coalesced pass
  // over the flattened [B, max_blocks] table, loads batched per thread.
  int bad = 0;
  const int nent = a.B * a.max_blocks;  // < 2^31, checked on the host
  constexpr int kBatch = 8;
  for (int e0 = threadIdx.x; e0 < nent; e0 += kBatch * blockDim.x) {
    int v[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int e = e0 + k * blockDim.x;
      v[k] = e < nent ? a.tables[e] : 0;
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int e = e0 + k * blockDim.x;
      if (e < nent) {
        const int b = e / a.max_blocks, i = e - b * a.max_blocks;
        if (i < s_nb[b] && (v[k] < 0 || v[k] >= a.num_blocks)) bad = 1;
      }
    }
  }
  // Each thread owns a contiguous run of sequences.
  const int per = ceil_div(a.B, blockDim.x);
  const int b0 = min(a.B, (int)threadIdx.x * per), b1 = min(a.B, b0 + per);
  int nfree = 0, nalloc = 0, nkept = 0;
  for (int b = b0; b < b1; ++b) {
    const int old_len = a.seq_lens[b];
    const int base = a.base_len ? a.base_len[b] : old_len;
    const int kept = a.keep[b] + a.keep_add;
    if (kept < 0 || kept > a.Kp1 || base < 0 || base > old_len || old_len < 0) { bad = 1; continue; }
    const int nb_old = ceil_div(old_len, bs), nb_new = ceil_div(base + kept, bs);
    if (nb_old > a.max_blocks || nb_new > a.max_blocks) { bad = 1; continue; }
    nfree += max(0, nb_old - nb_new);
    nalloc += max(0, nb_new - nb_old);
    nkept += kept;
  }
  if (bad) atomicOr(&s_bad, 1);
  int F, A, KT;
  const int fpre = block_excl_scan(nfree, &F);
  const int apre = block_excl_scan(nalloc, &A);
  const int kpre = block_excl_scan(nkept, &KT);
  const int ft = *a.free_top;
  if (threadIdx.x == 0) {
    if (s_bad || ft < 0 || ft > a.num_blocks || ft + F > a.num_blocks) s_code = SPEC_EINVAL;
    else if (ft + F < A) s_code = SPEC_ENOBLOCKS;
  }
  __syncthreads();
  // Blocks handed out come from stack positions [ft + F - A, ft + F); the
  // ones below ft must be valid ids (the pushed ones were checked above).
  if (s_code == 0) {
    for (int p = max(0, ft + F - A) + threadIdx.x; p < ft; p += blockDim.x) {
      const int x = a.free_stack[p];
      if (x < 0 || x >= a.num_blocks) atomicOr(&s_bad, 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_code == 0 && s_bad) s_code = SPEC_EINVAL;
  __syncthreads();
  if (s_code != 0) {
    if (threadIdx.x == 0) set_status(a.status, s_code);
    return;
  }
  // Frees: push table tails in sequence order.
  int fpos = ft + fpre;
  for (int b = b0; b < b1; ++b) {
    const int old_len = a.seq_lens[b];
    const int base = a.base_len ? a.base_len[b] : old_len;
    const int kept = a.keep[b] + a.keep_add;
    const int nb_old = ceil_div(old_len, bs), nb_new = ceil_div(base + kept, bs);
    int32_t* tab = a.tables + (size_t)b * a.max_blocks;
    for (int i = nb_new; i < nb_old; ++i) {
      a.free_stack[fpos++] = tab[i];
      tab[i] = -1;
    }
  }
  __syncthreads();
  // Allocations: pop from the top in sequence order; then lengths, offsets.
  const int top = ft + F;
  int k = apre, off = kpre;
  for (int b = b0; b < b1; ++b) {
    const int old_len = a.seq_lens[b];
    const int base = a.base_len ? a.base_len[b] : old_len;
    const int kept = a.keep[b] + a.keep_add;
    const int nb_old = ceil_div(old_len, bs), nb_new = ceil_div(base + kept, bs);
    int32_t* tab = a.tables + (size_t)b * a.max_blocks;
    for (int i = nb_old; i < nb_new; ++i) tab[i] = a.free_stack[top - 1 - (k++)];
    if (a.hid_off) a.hid_off[b] = off;
    off += kept;
  }
  __syncthreads();  // every read of seq_lens / base_len is done
  for (int b = b0; b < b1; ++b) {
    const int base = a.base_len ? a.base_len[b] : a.seq_lens[b];
    a.seq_lens[b] = base + a.keep[b] + a.keep_add;
  }
  if (threadIdx.x == 0) {
    *a.free_top = top - A;
    if (a.hid_off) a.hid_off[a.B] = KT;
  }
}

// Copy of kept token rows: a grid-stride loop over (token, part) items; the
// staged K/V segments of a token are split into kCopyParts parts.
__global__ void __launch_bounds__(kCopyThreads) commit_copy_kernel(CommitArgs a) {
  grid_dependency_wait();
  if (a.status && *(volatile int32_t*)a.status != SPEC_OK) return;
  const int nitems = a.B * a.Kp1 * kCopyParts;
  const int nseg = a.layers * 2;
  const int segs_per = (nseg + kCopyParts - 1) / kCopyParts;
  const int vps = a.seg_bytes / 16;  // vectors per segment
  for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
    const int tok = item / kCopyParts, part = item - tok * kCopyParts;
    const int b = tok / a.Kp1, i = tok - b * a.Kp1;
    const int kept = a.keep[b] + a.keep_add;
    if (i >= kept) continue;
    const int pos = a.seq_lens[b] - kept + i;  // base_len + i
    if (a.kv_stage) {
      const int blk = a.tables[(size_t)b * a.max_blocks + pos / a.block_size];
      const int slot = pos % a.block_size;
      const int s0 = part * segs_per, s1 = min(nseg, s0 + segs_per);
      const int nvec = max(0, s1 - s0) * vps;
      const uint4* src = reinterpret_cast<const uint4*>(
          a.kv_stage + (((size_t)b * a.Kp1 + i) * nseg + s0) * (size_t)a.seg_bytes);
      for (int v0 = threadIdx.x; v0 < nvec; v0 += blockDim.x * 4) {
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * blockDim.x;
          if (v < nvec) r[u] = __ldcs(src + v);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * blockDim.x;
          if (v < nvec) {
            const int seg = s0 + v / vps, e = v - (seg - s0) * vps;
            uint4* dst = reinterpret_cast<uint4*>(
                a.kv_pool + (((size_t)blk * nseg + seg) * a.block_size + slot) * (size_t)a.seg_bytes);
            __stcs(dst + e, r[u]);
          }
        }
      }
    }
    if (a.hid_stage && part == 0) {
      const int hv = a.hid_bytes / 16;
      const uint4* src =
          reinterpret_cast<const uint4*>(a.hid_stage + ((size_t)b * a.Kp1 + i) * a.hid_bytes);
      uint4* dst = reinterpret_cast<uint4*>(a.hid_out + (size_t)(a.hid_off[b] + i) * a.hid_bytes);
      for (int v = threadIdx.x; v < hv; v += blockDim.x) __stcs(dst + v, __ldcs(src + v));
    }
  }
}

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)a.B * sizeof(int);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(commit_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return cudaGetLastError();
  cudaError_t e = launch_pdl(commit_plan_kernel, dim3(1), dim3(kPlanThreads), smem, st, a);
  if (e != cudaSuccess) return e;
  if (a.B > 0 && a.Kp1 > 0 && (a.kv_stage || a.hid_stage)) {
    const int items = a.B * a.Kp1 * kCopyParts;
    e = launch_pdl(commit_copy_kernel, dim3(min(items, 148 * 4)), dim3(kCopyThreads), 0, st, a);
  }
  return e;
}

// ---------------------------------------------------------------------------
// Diagnostic: device Philox uniforms.
// ---------------------------------------------------------------------------
__global__ void philox_kernel(uint64_t seed, const uint32_t* ctr, int n, float* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float2 u = spec_uniforms(seed, ctr[4 * i], ctr[4 * i + 1], ctr[4 * i + 2], ctr[4 * i + 3]);
  out[2 * i] = u.x;
  out[2 * i + 1] = u.y;
}

cudaError_t launch_philox(uint64_t seed, const uint32_t* ctr, int n, float* out, cudaStream_t st) {
  if (n > 0) philox_kernel<<<(n + 255) / 256, 256, 0, st>>>(seed, ctr, n, out);
  return cudaGetLastError();
}

}  // namespace specv
