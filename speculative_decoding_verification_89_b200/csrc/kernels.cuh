// Internal interface between the C ABI and the kernels of libspecverify.
#pragma once

#include "common.cuh"

namespace specv {

// A logit row as the row-statistics kernel sees it.
struct RowRef {
  const unsigned char* ptr;  // first element of the row
  float T;                   // temperature of its sequence
  bool valid;                // statistics wanted (and temperature valid)
};

__device__ __forceinline__ RowRef make_row(const unsigned char* ptr, float T, bool want) {
  RowRef r;
  r.ptr = ptr;
  r.T = T;
  r.valid = want && temp_valid(T);
  return r;
}

// Each Rows type also names its "late" rows: those of positions below
// late_pos, which the draw after the check is most likely to read again (the
// first rejection falls at position j with probability decreasing in j). The
// row-statistics kernel streams them last so they are still in L2.

// Chain verification rows, grouped by sequence: for sequence b, rows
// b*(2K+1) + j are target row j (j <= K) and then draft row j - K - 1.
struct ChainRows {
  static constexpr bool kEntropy = false;
  const unsigned char* tgt;
  const unsigned char* drf;
  long long ld_tgt, ld_drf;  // row strides in bytes
  const float* temperature;
  int K;
  int late_pos;
  __device__ __forceinline__ bool late(int r) const {
    const int per = 2 * K + 1, j = r % per;
    return (j <= K ? j : j - K - 1) < late_pos;
  }
  __device__ __forceinline__ RowRef get(int r) const {
    const int per = 2 * K + 1, b = r / per, j = r - b * per;
    const float T = __ldg(temperature + b);
    if (j <= K) return make_row(tgt + ((long long)b * (K + 1) + j) * ld_tgt, T, true);
    return make_row(drf + ((long long)b * K + (j - K - 1)) * ld_drf, T, T != 0.0f);
  }
};

// Stage one of the two-stage check: per sequence, L_i rows at slots
// w .. w+K, then L_d rows at slots w .. w+K-1 (w = window length).
struct Hier1Rows {
  static constexpr bool kEntropy = false;
  const unsigned char* lg_i;
  const unsigned char* lg_d;
  long long ld;  // bytes
  const float* temperature;
  const int32_t* win_len;
  int K, S, Ni;
  int late_pos;
  __device__ __forceinline__ bool late(int r) const {
    const int per = 2 * K + 1, j = r % per;
    return (j <= K ? j : j - K - 1) < late_pos;
  }
  __device__ __forceinline__ RowRef get(int r) const {
    const int per = 2 * K + 1, b = r / per, j = r - b * per;
    const float T = __ldg(temperature + b);
    const int w = win_len[b];
    const bool ok = (w >= 0 && w < Ni);
    if (j <= K)
      return make_row(lg_i + ((long long)b * S + (ok ? w : 0) + j) * ld, T, ok);
    return make_row(lg_d + ((long long)b * S + (ok ? w : 0) + (j - K - 1)) * ld, T,
                    ok && T != 0.0f);
  }
};

// Stage two: L_f rows at slots 0 .. W of sequences whose window holds
// W >= Ni tokens after stage one (rows b*S + s).
struct Hier2Rows {
  static constexpr bool kEntropy = false;
  const unsigned char* lg_f;
  long long ld;
  const float* temperature;
  const int32_t* win_len;
  const int32_t* acc1;
  int S, Ni;
  int late_pos;
  __device__ __forceinline__ bool late(int r) const { return r % S < late_pos; }
  __device__ __forceinline__ RowRef get(int r) const {
    const int b = r / S, s = r - b * S;
    const int W = win_len[b];
    const bool fire = acc1[b] >= 0 && W >= Ni && W < S && s <= W;
    return make_row(lg_f + (long long)r * ld, __ldg(temperature + b), fire);
  }
};

// Draft step: row b of the drafting exit's logits, one row per sequence; the
// row statistics also gather the first moment the entropy needs.
struct DraftRows {
  static constexpr bool kEntropy = true;
  const unsigned char* lg;
  long long ld;  // bytes
  const float* temperature;
  __device__ __forceinline__ bool late(int) const { return false; }
  __device__ __forceinline__ RowRef get(int r) const {
    return make_row(lg + (long long)r * ld, __ldg(temperature + r), true);
  }
};

// Workspace pieces of the row-statistics step.
struct RsBuffers {
  Partial* part;    // [rows, tiles]
  double* mom;      // [rows, tiles] first moments (Rows::kEntropy only)
  int32_t* zero;    // optional word set to 0 once the launch may write (a ticket of a later launch)
};

// Combine a row's tile partials (warp-cooperative; result valid in lane 0).
// Up to 4*32 tiles are read once into registers; longer rows loop. s_out, if
// given, gets the sum 2^L itself (0 where it is not formed).
__device__ __forceinline__ RowFinal combine_row(const Partial* p, int ntiles, bool greedy,
                                                float chi, int lane, double* s_out = nullptr) {
  constexpr int kReg = 4;
  float pm[kReg];
  double ps[kReg];
  int pi[kReg];
#pragma unroll
  for (int k = 0; k < kReg; ++k) {
    const int t = lane + 32 * k;
    if (t < ntiles) {
      const Partial q = p[t];
      pm[k] = q.m;
      pi[k] = q.idx;
      ps[k] = q.s;
    } else {
      pm[k] = -INFINITY;
      pi[k] = 0x7fffffff;
      ps[k] = 0.0;
    }
  }
  float mv = -INFINITY;
  int mi = 0x7fffffff;
#pragma unroll
  for (int k = 0; k < kReg; ++k)
    if (pm[k] > mv || (pm[k] == mv && pi[k] < mi)) { mv = pm[k]; mi = pi[k]; }
  for (int t = lane + 32 * kReg; t < ntiles; t += 32) {
    const float m = p[t].m;
    const int i = p[t].idx;
    if (m > mv || (m == mv && i < mi)) { mv = m; mi = i; }
  }
  warp_argmax(mv, mi);
  RowFinal f;
  f.m = mv;
  f.amax = mi;
  f.M = 0.0;
  f.L = 0.0;
  f.pad = 0;
  bool ok = (mv > -INFINITY && mv < INFINITY);
  if (ok && !greedy) {
    f.M = (double)__fmul_rn(mv, chi);
    double s = 0.0;
#pragma unroll
    for (int k = 0; k < kReg; ++k)
      if (ps[k] != 0.0) s += ps[k] * exp2((double)__fmul_rn(pm[k], chi) - f.M);
    for (int t = lane + 32 * kReg; t < ntiles; t += 32) {
      const double st = p[t].s;
      if (st != 0.0) s += st * exp2((double)__fmul_rn(p[t].m, chi) - f.M);
    }
    s = warp_sum_d(s);
    ok = (s > 0.0 && s < INFINITY);
    f.L = log2(s);
    if (s_out) *s_out = s;
  }
  f.ok = ok;
  return f;
}


template <typename Rows>
cudaError_t launch_row_stats(int dtype, const Rows& rows, int nrows, int V, const RsBuffers& b,
                             int32_t* status, cudaStream_t st);

// ----------------------------------------------------------------------------
// Decide kernels (accept test, first rejection, residual / bonus draw)
// ----------------------------------------------------------------------------
struct DecideCommon {
  int dtype, B, K, V;
  const int32_t* draft_tok;
  const float* temperature;
  uint64_t seed;
  const int32_t* seq_id;
  uint32_t round;
  const Partial* part;             // [rows, ntiles] tile partials
  int ntiles;
  RowFinal* fin;                   // [rows] final row statistics
  double* diag;
  int32_t* status;
};

struct ChainDecideArgs {
  DecideCommon c;
  const unsigned char* tgt;
  const unsigned char* drf;
  long long ld_tgt, ld_drf;        // bytes
  int32_t* accept_len;
  int32_t* out_tok;
};

struct HierDecideArgs {
  DecideCommon c;
  const unsigned char* lg_d;
  const unsigned char* lg_i;
  const unsigned char* lg_f;
  long long ld;                    // bytes
  int S, Ni;
  int32_t* win_len;
  int32_t* win_tok;
  double* win_stat;                // [B, Ni+K, 2]: (row max, ln sum exp((l-max)/T))
  int32_t* acc1;
  int32_t* acc2;
  int32_t* commit_tok;
  int32_t* commit_n;
};

cudaError_t launch_chain_decide(const ChainDecideArgs& a, cudaStream_t st);
cudaError_t launch_hier1_decide(const HierDecideArgs& a, cudaStream_t st);
cudaError_t launch_hier2_decide(const HierDecideArgs& a, cudaStream_t st);
__host__ __device__ __forceinline__ int residual_tiles(int V) {  // kResTile tiles per row
  return (V + kResTile - 1) / kResTile;
}

// ----------------------------------------------------------------------------
// Vocabulary-parallel chain verification (vocab.cu)
// ----------------------------------------------------------------------------
// One row's statistics over one vocabulary shard [v0, v0 + Vs): the shard's
// largest logit m and its global id, the shift M = fl(m * c_hi) and
// S = sum over the shard of 2^(l*c - M), and the logit x of the row's
// drafted token when the shard holds it. 32 bytes, exchanged between ranks.
constexpr int kVpHasX = 1;  // the shard holds the drafted token: x is its logit
constexpr int kVpBad = 2;   // the shard saw a NaN or +inf logit
struct VpRow {
  double M, S;
  float m;
  int amax;
  float x;
  int flags;
};
static_assert(sizeof(VpRow) == SPEC_VP_ROW_BYTES, "record size is part of the C ABI");
// One sequence's draw weights over one shard: z = the shard's sum of the
// weights of the draw (max(0, p - q) at a rejection, p for the bonus token),
// p = the shard's mass under the target row of the draw.
struct VpMass {
  double z, p;
};
static_assert(sizeof(VpMass) == SPEC_VP_MASS_BYTES, "record size is part of the C ABI");
// What the decide launch leaves for the pick launch, per sequence.
struct VpSeq {
  double Lp, Lq;  // log2-partitions of the draw's target / draft rows
  float mp, mq;   // their largest logits
  float u;        // draw uniform
  int a;          // first rejection (K: all accepted)
  int state;      // kVpSeqBad, kVpSeqGreedy or kVpSeqDraw
  int tok;        // greedy: the token at a
};
constexpr int kVpSeqBad = 0, kVpSeqGreedy = 1, kVpSeqDraw = 2;

struct VpArgs {
  int B, K, Vs, v0, V, R, rank;
  const unsigned char* tgt;   // this rank's shard rows
  const unsigned char* drf;
  long long ld_tgt, ld_drf;   // bytes
  const int32_t* draft_tok;
  const float* temperature;
  uint64_t seed;
  const int32_t* seq_id;
  uint32_t round;
  const Partial* part;        // row-statistics partials of the shard rows
  int ntiles;
  VpRow* rows;                // [B, 2K+1] this rank's records
  const VpRow* rows_all;      // [R, B, 2K+1] every rank's, in rank order
  VpMass* mass;               // [B] this rank's
  const VpMass* mass_all;     // [R, B]
  VpSeq* seq;                 // [B]
  double* tsum;               // [B, nrt] residual tile sums of the shard
  double* pre;                // [B, nrt] their prefixes
  int32_t* accept_len;
  int32_t* out_tok;
  double* diag;
  int32_t* status;
};
cudaError_t launch_vp_records(int dtype, const VpArgs& a, cudaStream_t st);
cudaError_t launch_vp_decide(int dtype, const VpArgs& a, cudaStream_t st);
cudaError_t launch_vp_pick(int dtype, const VpArgs& a, cudaStream_t st);

// ----------------------------------------------------------------------------
// Paged commit
// ----------------------------------------------------------------------------
struct CommitArgs {
  int B, block_size, max_blocks, num_blocks, Kp1, keep_add;
  int32_t* tables;
  int32_t* seq_lens;
  const int32_t* base_len;
  const int32_t* keep;
  int32_t* free_stack;
  int32_t* free_top;
  const unsigned char* kv_stage;
  unsigned char* kv_pool;
  int layers, seg_bytes;           // seg_bytes = kv_heads * head_dim * 2
  const unsigned char* hid_stage;
  unsigned char* hid_out;
  int32_t* hid_off;
  int hid_bytes;                   // hidden * 2
  int32_t* status;
};

// One sequence's part of a commit plan, formed before the planner runs.
constexpr int kRecTail = 4;
struct CommitRec {
  int held;  // table entries held: min(blocks of the old length, max_blocks)
  int len;   // new length base + kept; -1 if an input of the sequence or a held entry is invalid
  int kept;
  int pad;
  int tail[kRecTail];  // the first table entries to be freed (-1 past the last)
};
static_assert(sizeof(CommitRec) == 32, "two 16-byte stores");

// The planner launch, then the copy launch; the copy launch alone.
cudaError_t launch_commit(const CommitArgs& a, cudaStream_t st);
cudaError_t launch_commit_copy(const CommitArgs& a, cudaStream_t st);
// The copy launch of the verify-and-commit path: it starts its copies once
// *plan_flag is nonzero (set by the planner of the decide launch before it).
cudaError_t launch_commit_copy_planned(const CommitArgs& a, const int32_t* plan_flag,
                                       cudaStream_t st);

// ----------------------------------------------------------------------------
// Chain verification fused with the paged commit of its kept rows
// ----------------------------------------------------------------------------
struct FusedArgs {
  ChainDecideArgs d;
  CommitArgs cm;       // keep = d.accept_len, keep_add = 1, Kp1 = K + 1
  int32_t* ticket;     // zeroed by the row-statistics launch that precedes this call
  int32_t* plan_flag;  // 0 at the decide launch's start, 1 once its planner has run
  CommitRec* rec;      // [B] per-sequence records for the planner
};

// The decide launch that also plans the commit, then the copy launch; the
// row statistics precede.
cudaError_t launch_chain_fused(const FusedArgs& a, cudaStream_t st);

// SPEC_OK for cudaSuccess; otherwise records e as the calling thread's last
// CUDA error (spec_last_cuda_error) and returns SPEC_ECUDA.
int record_cuda_status(cudaError_t e);

// ----------------------------------------------------------------------------
// Chain verification step: one persistent launch for the row statistics, the
// checks, the draws and (optionally) the paged commit, after a prologue launch
// that clears its counters.
// ----------------------------------------------------------------------------
constexpr int kChunkTiles = 4;   // tiles per stream chunk of an early row (about)
constexpr int kLateChunkTiles = 2;  // tiles per stream chunk of a late row (about)
constexpr int kCopyUnit = 8192;  // bytes of K/V rows per copy unit
constexpr int kPartBytes = 4096;  // bytes of each row per draw part
__host__ __device__ constexpr int part_tiles(int esz) { return kPartBytes / (256 * esz); }

// Statistics of one chunk of consecutive tiles of one row. Sampled rows:
// largest raw logit m, the exact fp32 shift M (as bits in aux) the chunk's
// sum s = sum 2^(l*c - M) is taken against. Greedy rows: m and its first
// index (aux); s = 0.
struct ChunkStat {
  float m;
  int aux;
  double s;
};

// Per-call counters, cleared by the prologue launch.
struct StepCounters {
  unsigned stream;  // next stream item
  unsigned draw;    // next draw part
  unsigned copy;    // next copy unit
  int ticket;       // sequences whose check is done
  int plan;         // 0 pending, 1 commit planned, 2 nothing to copy
  int abort;        // a bounded wait gave up: the other waits stop too
  int kt;           // kept tokens of the planned commit
  int pad;
};

// What a sequence's check leaves for its draw and its commit.
constexpr int kSeqDraw = 1;  // a token is to be drawn (sampled, valid)
constexpr int kSeqHasQ = 2;  // the draw is a residual (a < K): draft row a exists
struct SeqState {
  double lt, lq;  // log2-partitions of target row a and draft row a
  float mt, mq;   // their largest logits
  float u;        // draw uniform of position a
  int a;          // accepted drafts (-1: invalid sequence)
  int flags;
  int old_len, base, kept, bad;  // commit: lengths before, kept rows, checks failed
  int pad;
};

struct StepArgs {
  int dtype, B, K, V;
  const unsigned char* tgt;
  const unsigned char* drf;
  long long ld_tgt, ld_drf;  // bytes
  const int32_t* draft_tok;
  const float* temperature;
  uint64_t seed;
  const int32_t* seq_id;
  uint32_t round;
  int32_t* accept_len;
  int32_t* out_tok;
  double* diag;
  int32_t* status;
  // schedule: nt tiles per row; rows of positions < lp ("late") are streamed
  // after all others, in NCl chunks each, the others in NCe chunks (re early
  // and rl late row slots per sequence); chunk statistics have a row stride
  // of NC = max(NCe, NCl)
  int nt, NC, NCe, NCl, lp, re, rl;
  unsigned n_early, n_total;  // stream items
  int nrt, D;                 // residual tiles per row, draw parts (part_tiles tiles) per sequence
  // workspace
  ChunkStat* part;  // [B * (2K+1)][NC]
  RowFinal* fin;    // [B * (2K+1)] row statistics
  SeqState* seq;    // [B]
  double* tsum;     // [B][nrt] residual tile sums
  double* ptot;     // [B][D] draw-part totals
  StepCounters* ctr;
  int* row_cnt;     // [B * (2K+1)] chunks done
  int* seq_cnt;     // [B] rows done
  int* seq_done;    // [B] check done
  int* draw_cnt;    // [B] draw parts done
  int* tok_seq;     // [B * (K+1)] sequence of each kept token
  int* tok_off;     // [B] first kept token of each sequence
  // commit (commit != 0)
  int commit;
  int unit_segs, units_kv, units_tok;  // K/V segments per copy unit; units per token
  CommitArgs cm;
};

cudaError_t launch_chain_step(const StepArgs& a, cudaStream_t st);

// Saguaro sampling: T ln(1 - eps) added in place to the cached tokens' logits
// of each sequence's draft rows (see saguaro.cu).
cudaError_t launch_saguaro_adjust(int dtype, unsigned char* lg, long long ld_bytes, int B,
                                  int rows_per_seq, int V, const int32_t* cached, int n_cached,
                                  int per_row, double ln1m_eps, const float* temperature,
                                  cudaStream_t st);

cudaError_t launch_philox(uint64_t seed, const uint32_t* ctr, int n, float* out, cudaStream_t st);

// Outcome law of a chain check (drafts fixed): see outcome.cu.
struct OutcomeArgs {
  int B, K, V, n_top, ntiles;
  int late_pos;         // row pairs k < late_pos were streamed last by the statistics
  const unsigned char* tgt;
  const unsigned char* drf;
  long long ld_tgt, ld_drf;  // bytes
  const int32_t* draft_tok;
  const float* temperature;
  const Partial* part;  // [B * (2K+1), ntiles]
  double* zk;           // [B, K+1] residual masses
  double* lt;           // [B, 2K+1] row log2-partitions (NaN: no finite statistics)
  double* cw;           // [B, K+1, n_top] best weights (fp64)
  int* cv;              // [B, K+1, n_top] their tokens
  double* p_len;        // out [B, K+1]
  double* beta;         // out [B, K] or null
  double* mass;         // out [B, K+1] or null
  int32_t* top_len;     // out [B, n_top]
  int32_t* top_tok;     // out [B, n_top]
  double* top_prob;     // out [B, n_top]
  int32_t* status;
};
cudaError_t launch_outcome(int dtype, const OutcomeArgs& a, cudaStream_t st);

// Draft step over B rows of the drafting exit: row statistics with the first
// moments, then one cluster per sequence for the entropy and the draw.
cudaError_t launch_draft_step(int dtype, const unsigned char* lg, long long ld_bytes, int B, int V,
                              const float* temperature, uint64_t seed, const int32_t* seq_id,
                              uint32_t round, const int32_t* pos, Partial* part, double* mom,
                              int32_t* out_tok, double* out_logq, double* out_entropy,
                              int32_t* status, cudaStream_t st);



}  // namespace specv
