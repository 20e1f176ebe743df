// Paged-commit bodies shared by the commit launches and the fused
// verify-and-commit path: the planner (one CTA) and the row copy (many CTAs).
// HiSpec (gist.science summary of arXiv 2510.01336), section 2: buffered KV
// entries and hidden states of rejected tokens are dropped before the next
// phase; block tables let every sequence keep its own number of tokens.
#pragma once
#include "common.cuh"
#include "kernels.cuh"

namespace specv {

constexpr int kPlanThreads = 1024;
constexpr int kCopyThreads = 256;
constexpr int kCopyCtasPerSm = 8;  // 64 warps per SM: one round of items for most calls
// The copy launch that starts beside the decide launch finds room for few CTAs
// until the decide CTAs leave; 6 per SM measured best there (B=64, K=8,
// V=128256 bf16 step: 78.8 us, against 79.4 at 5, 79.7 at 7, 80.4 at 4 and
// 8 per SM), 8 after a plain planner launch.
constexpr int kCopyCtasPerSmPlanned = 6;

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Block-wide exclusive scan of four ints per thread (any block of up to 1024
// threads, a multiple of 32); totals returned in tot.
static __device__ int4 block_excl_scan4(int4 v, int4* tot) {
  __shared__ int4 warp_sums[32];
  __shared__ int4 s_tot;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int4 incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yx = __shfl_up_sync(0xffffffffu, incl.x, o);
    const int yy = __shfl_up_sync(0xffffffffu, incl.y, o);
    const int yz = __shfl_up_sync(0xffffffffu, incl.z, o);
    const int yw = __shfl_up_sync(0xffffffffu, incl.w, o);
    if (lane >= o) { incl.x += yx; incl.y += yy; incl.z += yz; incl.w += yw; }
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int4 w = lane < (int)(blockDim.x >> 5) ? warp_sums[lane] : make_int4(0, 0, 0, 0);
    int4 wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int yx = __shfl_up_sync(0xffffffffu, wi.x, o);
      const int yy = __shfl_up_sync(0xffffffffu, wi.y, o);
      const int yz = __shfl_up_sync(0xffffffffu, wi.z, o);
      const int yw = __shfl_up_sync(0xffffffffu, wi.w, o);
      if (lane >= o) { wi.x += yx; wi.y += yy; wi.z += yz; wi.w += yw; }
    }
    warp_sums[lane] = make_int4(wi.x - w.x, wi.y - w.y, wi.z - w.z, wi.w - w.w);  // exclusive
    if (lane == 31) s_tot = wi;
  }
  __syncthreads();
  const int4 base = warp_sums[warp];
  *tot = s_tot;
  return make_int4(base.x + incl.x - v.x, base.y + incl.y - v.y, base.z + incl.z - v.z,
                   base.w + incl.w - v.w);
}

// One CTA. Two rounds of global reads: (1) the per-sequence lengths and
// counts, (2) after a block scan, every covered table entry (validation), the
// tails to be freed and the stack entries to be popped below the old top,
// the last two cached in shared memory. Every check is made before anything
// is written; the writes then need no further reads while the caches hold.
constexpr int kPushCache = 2048;   // freed entries cached in push order
constexpr int kStackCache = 2048;  // stack entries popped from below the old top

// One sequence's part of the plan, formed by a CTA of its own before the
// planner runs (the verify-and-commit decide launch's leader of the sequence,
// once its accept test is done): the table entries it holds, checked, its new
// length and the first entries to be freed. The planner then reads one record
// per sequence instead of the lengths and the whole table row. The record's
// layout, CommitRec, is declared with CommitArgs.

// Whole CTA; old_len = seq_lens[b]. The checks are plan_body's, per sequence.
static __device__ void commit_record(const CommitArgs& a, int b, int old_len, int kept,
                                     CommitRec* out) {
  __shared__ int s_tail[kRecTail];
  const int base = a.base_len ? a.base_len[b] : old_len;
  const int bs = a.block_size;
  const int nbo = ceil_div(max(old_len, 0), bs);
  int nbn = nbo;
  bool ok = !(kept < 0 || kept > a.Kp1 || base < 0 || base > old_len || old_len < 0);
  if (ok) {
    nbn = ceil_div(base + kept, bs);
    if (nbo > a.max_blocks || nbn > a.max_blocks) ok = false;
  }
  const int held = min(nbo, a.max_blocks);
  const int32_t* tab = a.tables + (size_t)b * a.max_blocks;
  int bad = 0;
  for (int i = threadIdx.x; i < held; i += blockDim.x) {
    const int v = tab[i];
    if (v < 0 || v >= a.num_blocks) bad = 1;
    if (i >= nbn && i < nbn + kRecTail) s_tail[i - nbn] = v;
  }
  bad = __syncthreads_or(bad);
  if (threadIdx.x == 0) {
    const bool good = ok && !bad;
    const int4 h = make_int4(held, good ? base + kept : -1, kept, 0);
    int t[kRecTail];
#pragma unroll
    for (int j = 0; j < kRecTail; ++j) t[j] = (good && nbn + j < held) ? s_tail[j] : -1;
    reinterpret_cast<int4*>(out)[0] = h;
    reinterpret_cast<int4*>(out)[1] = make_int4(t[0], t[1], t[2], t[3]);
  }
}

// s_seq: dynamic shared memory of 3 * B ints. Runs in any block of up to 1024
// threads. The kept counts are read from L2: in the fused verify-and-commit
// path they were written by other CTAs of the same grid. With recs (one
// CommitRec per sequence, written by other CTAs of the same grid) the lengths,
// counts, table checks and the first freed entries come from the records.
static __device__ void plan_body(const CommitArgs& a, int* s_seq,
                                 const CommitRec* recs = nullptr) {
  // [3][B]: table-entry prefix, new length, kept
  int* s_nbp = s_seq;             // blocks held before, then their exclusive prefix
  int* s_len = s_seq + a.B;
  int* s_kept = s_seq + 2 * a.B;
  __shared__ int s_push[kPushCache];
  __shared__ int s_stack[kStackCache];
  __shared__ int s_bad, s_sbad, s_code, s_ft, s_st0;
  // One thread reads the status word (with the per-sequence inputs, not
  // before them) and the block acts on that one value, so the early return
  // below is taken by every thread or by none.
  if (threadIdx.x == 0) {
    s_st0 = a.status ? *(volatile int32_t*)a.status : SPEC_OK;
    s_bad = 0;
    s_sbad = 0;
    s_code = 0;
    s_ft = *a.free_top;
  }
  const int bs = a.block_size;
  // Each thread owns a contiguous run of sequences (sequence order matters
  // for the allocation order).
  const int per = ceil_div(a.B, blockDim.x);
  const int b0 = min(a.B, (int)threadIdx.x * per), b1 = min(a.B, b0 + per);
  int4 cnt = make_int4(0, 0, 0, 0);  // frees, allocations, kept rows, table entries
  int bad = 0;
  int4 tail0 = make_int4(-1, -1, -1, -1);  // record tail of the run's first sequence
  for (int b = b0; recs && b < b1; ++b) {
    const int4 h = __ldcg(reinterpret_cast<const int4*>(recs + b));
    if (b == b0) tail0 = __ldcg(reinterpret_cast<const int4*>(recs + b) + 1);
    const int held = h.x, len = h.y, kept = h.z;
    if (len < 0) bad = 1;
    const int nbn = len < 0 ? held : ceil_div(len, bs);
    s_nbp[b] = held;
    s_len[b] = len < 0 ? 0 : len;
    s_kept[b] = kept;
    cnt.x += max(0, held - nbn);
    cnt.y += max(0, nbn - held);
    cnt.z += kept;
    cnt.w += held;
  }
  for (int b = b0; !recs && b < b1; ++b) {
    const int old_len = a.seq_lens[b];
    const int base = a.base_len ? a.base_len[b] : old_len;
    const int kept = __ldcg(a.keep + b) + a.keep_add;
    int nbo = ceil_div(max(old_len, 0), bs), nbn = nbo;
    bool ok = true;
    if (kept < 0 || kept > a.Kp1 || base < 0 || base > old_len || old_len < 0) {
      ok = false;
    } else {
      nbn = ceil_div(base + kept, bs);
      if (nbo > a.max_blocks || nbn > a.max_blocks) ok = false;
    }
    if (!ok) bad = 1;
    const int held = min(nbo, a.max_blocks);
    s_nbp[b] = held;
    s_len[b] = ok ? base + kept : 0;
    s_kept[b] = kept;
    cnt.x += max(0, nbo - nbn);
    cnt.y += max(0, nbn - nbo);
    cnt.z += kept;
    cnt.w += held;
  }
  __syncthreads();  // publishes s_st0
  if (s_st0 != SPEC_OK) return;  // sticky error: one value for every thread
  if (bad) atomicOr(&s_bad, 1);
  int4 tot;
  const int4 pre = block_excl_scan4(cnt, &tot);  // its barriers also publish s_ft, s_bad
  {
    int q = pre.w;  // blocks held -> their exclusive prefix, over this thread's run
    for (int b = b0; b < b1; ++b) {
      const int h = s_nbp[b];
      s_nbp[b] = q;
      q += h;
    }
  }
  const int F = tot.x, A = tot.y, KT = tot.z, NE = tot.w, ft = s_ft;
  auto held = [&](int b) { return (b + 1 < a.B ? s_nbp[b + 1] : NE) - s_nbp[b]; };
  __syncthreads();
  const bool sizes_ok = !s_bad && ft >= 0 && ft <= a.num_blocks && ft + F <= a.num_blocks;
  // Pops come from stack positions [lo, ft + F): those at or above ft are the
  // entries pushed by this call, those below ft are read here.
  const int lo = max(0, ft + F - A);
  const bool cached = F <= kPushCache && ft - lo <= kStackCache;
  if (sizes_ok) {
    // Every covered table entry must be a valid block id (the records' CTAs
    // checked them already): 1, 2 or 4 sequences per warp (32, 16 or 8 lanes
    // each), 16 loads in flight per lane.
    if (!recs) {
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
      const int need = ceil_div(a.B, nwarps);
      const int spw = need <= 1 ? 1 : (need <= 2 ? 2 : 4);
      const int lps = 32 / spw, sub = lane / lps, sl = lane % lps;
      constexpr int kBatch = 16;
      for (int bb = warp * spw; bb < a.B; bb += nwarps * spw) {
        const int b = bb + sub;
        const int nb = b < a.B ? held(b) : 0;
        const int32_t* tab = a.tables + (size_t)(b < a.B ? b : 0) * a.max_blocks;
        for (int i0 = sl; i0 < nb; i0 += lps * kBatch) {
          int v[kBatch];
#pragma unroll
          for (int k = 0; k < kBatch; ++k) v[k] = (i0 + lps * k < nb) ? tab[i0 + lps * k] : 0;
#pragma unroll
          for (int k = 0; k < kBatch; ++k)
            if (i0 + lps * k < nb && (v[k] < 0 || v[k] >= a.num_blocks)) bad = 1;
        }
      }
    }
    // Tails to be freed, cached in push order (same round of reads).
    if (cached) {
      int fpos = pre.x;
      for (int b = b0; b < b1; ++b) {
        const int32_t* tab = a.tables + (size_t)b * a.max_blocks;
        const int nbn = ceil_div(s_len[b], bs);
        for (int i = nbn; i < held(b); ++i) {
          const int j = i - nbn;
          int v;
          if (!recs || j >= kRecTail) v = tab[i];
          else if (b == b0) v = j == 0 ? tail0.x : j == 1 ? tail0.y : j == 2 ? tail0.z : tail0.w;
          else v = __ldcg(&recs[b].tail[j]);
          s_push[fpos++] = v;
        }
      }
    }
    if (bad) atomicOr(&s_bad, 1);
    // Stack entries popped from below the old top must be valid ids.
    int sbad = 0;
    for (int p = lo + threadIdx.x; p < ft; p += blockDim.x) {
      const int x = a.free_stack[p];
      if (x < 0 || x >= a.num_blocks) sbad = 1;
      if (cached) s_stack[p - lo] = x;
    }
    if (sbad) atomicOr(&s_sbad, 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // the order of the checks fixes which status wins
    if (!sizes_ok || s_bad) s_code = SPEC_EINVAL;
    else if (ft + F < A) s_code = SPEC_ENOBLOCKS;
    else if (s_sbad) s_code = SPEC_EINVAL;
  }
  __syncthreads();
  if (s_code != 0) {
    if (threadIdx.x == 0) set_status(a.status, s_code);
    return;
  }
  // Frees: push table tails in sequence order.
  int fpos = pre.x;
  for (int b = b0; b < b1; ++b) {
    int32_t* tab = a.tables + (size_t)b * a.max_blocks;
    for (int i = ceil_div(s_len[b], bs); i < held(b); ++i) {
      a.free_stack[ft + fpos] = cached ? s_push[fpos] : tab[i];
      ++fpos;
      tab[i] = -1;
    }
  }
  if (!cached) __syncthreads();  // pops below read the pushed entries back
  // Allocations: pop from the top in sequence order; lengths and offsets.
  const int top = ft + F;
  int k = pre.y, off = pre.z;
  for (int b = b0; b < b1; ++b) {
    int32_t* tab = a.tables + (size_t)b * a.max_blocks;
    const int nbn = ceil_div(s_len[b], bs);
    for (int i = held(b); i < nbn; ++i) {
      const int p = top - 1 - (k++);
      tab[i] = !cached ? a.free_stack[p] : (p >= ft ? s_push[p - ft] : s_stack[p - lo]);
    }
    if (a.hid_off) a.hid_off[b] = off;
    off += s_kept[b];
    a.seq_lens[b] = s_len[b];
  }
  if (threadIdx.x == 0) {
    *a.free_top = top - A;
    if (a.hid_off) a.hid_off[a.B] = KT;
  }
}

// Copy of kept token rows. Every CTA scans the kept counts (the planner has
// checked them) so kept rows are numbered 0..KT-1; warps then stride over
// (kept row, segment) items. A segment is one (layer, K|V) slice of a token's
// staged row (kv_heads * head_dim * 2 bytes, contiguous in both stage and
// pool); the hidden row is cut into pieces of the same size after them.
// s_off: dynamic shared memory of 2 * B + 1 ints. CTA `cta` of `ncta` taking
// part; any block size that is a multiple of 32 and at least 64.
static __device__ void copy_body(const CommitArgs& a, int cta, int ncta, int* s_off) {
  // [B + 1] exclusive scan of kept rows, then [B] new lengths
  int* s_len = s_off + a.B + 1;
  // The status word is read (by one thread) with the counts, and checked by
  // every thread on that one value once they are in.
  __shared__ int s_st0;
  if (threadIdx.x == 0) s_st0 = a.status ? *(volatile int32_t*)a.status : SPEC_OK;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int b = (int)threadIdx.x - 32; b >= 0 && b < a.B; b += blockDim.x - 32)
    s_len[b] = __ldcg(a.seq_lens + b);  // the other warps, while warp 0 scans
  if (warp == 0) {
    int carry = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      const int v = b < a.B ? __ldcg(a.keep + b) + a.keep_add : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b < a.B) s_off[b] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[a.B] = carry;
  }
  __syncthreads();
  if (s_st0 != SPEC_OK) return;  // sticky error: one value for every thread
  const int KT = s_off[a.B];
  const int nseg = a.kv_stage ? a.layers * 2 : 0;
  const int piece = a.kv_stage ? a.seg_bytes : 2048;
  const int nhid = a.hid_stage ? (a.hid_bytes + piece - 1) / piece : 0;
  const int per_tok = nseg + nhid;
  const int nitems = KT * per_tok;
  const int nw = ncta * (blockDim.x >> 5);
  for (int item = cta * (blockDim.x >> 5) + warp; item < nitems; item += nw) {
    const int k = item / per_tok, sidx = item - k * per_tok;
    int lo = 0, hi = a.B - 1;  // the sequence b with s_off[b] <= k < s_off[b + 1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= k) lo = mid; else hi = mid - 1;
    }
    const int b = lo, i = k - s_off[b];
    const int kept = s_off[b + 1] - s_off[b];
    const uint4* src;
    uint4* dst;
    int nvec;
    if (sidx < nseg) {
      const int pos = s_len[b] - kept + i;  // base_len + i
      const int blk = __ldcg(a.tables + (size_t)b * a.max_blocks + pos / a.block_size);
      const int slot = pos % a.block_size;
      src = reinterpret_cast<const uint4*>(a.kv_stage +
                                           (((size_t)b * a.Kp1 + i) * nseg + sidx) * a.seg_bytes);
      dst = reinterpret_cast<uint4*>(
          a.kv_pool + (((size_t)blk * nseg + sidx) * a.block_size + slot) * (size_t)a.seg_bytes);
      nvec = a.seg_bytes / 16;
    } else {
      const int h = sidx - nseg;
      const int off = h * piece, len = min(piece, a.hid_bytes - off);
      src = reinterpret_cast<const uint4*>(a.hid_stage + ((size_t)b * a.Kp1 + i) * a.hid_bytes + off);
      dst = reinterpret_cast<uint4*>(a.hid_out + (size_t)(s_off[b] + i) * a.hid_bytes + off);
      nvec = len / 16;
    }
    for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
      uint4 r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (v0 + 32 * u < nvec) r[u] = __ldcs(src + v0 + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (v0 + 32 * u < nvec) __stcs(dst + v0 + 32 * u, r[u]);
    }
  }
}

}  // namespace specv
