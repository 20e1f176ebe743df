// C ABI of libspecverify: argument checks on the host, workspace carving and
// the launch sequence of each call. Declarations and the contract of every
// entry point are in include/spec_verify.h.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"

using namespace specv;

namespace specv {
// decide.cu: the chain check of V <= SPEC_SMALL_V in one launch, one CTA per
// sequence forming its rows' statistics itself.
cudaError_t launch_chain_small(const ChainDecideArgs& a, cudaStream_t st);
}  // namespace specv

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
bool aligned(const void* p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }
int elem_size(int dtype) { return dtype == SPEC_BF16 ? 2 : 4; }
int stat_tiles(int V, int dtype) {
  const int ept = kTileBytes / elem_size(dtype);
  return (V + ept - 1) / ept;
}

struct Layout {
  size_t part, fin, ticket, rec, seq, tsum, ctr, ints, total;
  long long rows;
};

// Workspace, each region 256-byte aligned: final row statistics and tile
// partials for the largest row set (the step kernel keeps its chunk
// statistics in the partials' place), the ticket and plan words and the
// per-sequence commit records of the staged verify-and-commit path, then the
// step kernel's per-sequence states,
// residual tile sums, counters and per-sequence integer arrays.
bool layout(int B, int K, int V, int dtype, int Ni, Layout* L) {
  if (B < 0 || K < 0 || K > SPEC_MAX_K || V < 1 || V > SPEC_MAX_V) return false;
  if (dtype != SPEC_F32 && dtype != SPEC_BF16) return false;
  if (Ni < 0 || Ni > SPEC_MAX_K) return false;
  const long long per = Ni > 0 ? (long long)std::max(2 * K + 1, Ni + K + 1) : 2LL * K + 1;
  const long long rows = (long long)B * per;
  if (rows * stat_tiles(V, dtype) >= (1LL << 31)) return false;  // 32-bit item indices
  L->rows = rows;
  L->fin = 0;
  L->part = align_up((size_t)rows * sizeof(RowFinal));
  L->ticket = L->part + align_up((size_t)rows * stat_tiles(V, dtype) * sizeof(Partial));
  L->rec = L->ticket + kAlign;
  L->seq = L->rec + align_up((size_t)B * sizeof(CommitRec));
  L->tsum = L->seq + align_up((size_t)B * sizeof(SeqState));
  // residual tile sums [B][nrt], then the draw-part totals [B][D]
  const size_t pt = part_tiles(elem_size(dtype));
  const size_t nrt = residual_tiles(V), D = (nrt + pt - 1) / pt;
  L->ctr = L->tsum + align_up((size_t)B * (nrt + D) * sizeof(double));
  L->ints = L->ctr + align_up(sizeof(StepCounters));
  // seq_cnt, seq_done, draw_cnt, tok_off [B] each; tok_seq [B * (K+1)]; row_cnt [rows]
  L->total = L->ints + align_up(((size_t)B * (4 + K + 1) + (size_t)rows) * sizeof(int));
  return true;
}

// Draft-step workspace: run partials and first moments of the B rows.
struct DraftLayout {
  size_t part, mom, total;
};
bool draft_layout(int B, int V, int dtype, DraftLayout* L) {
  if (B < 0 || V < 1 || V > SPEC_MAX_V) return false;
  if (dtype != SPEC_F32 && dtype != SPEC_BF16) return false;
  const long long n = (long long)B * stat_tiles(V, dtype);
  if (n >= (1LL << 31)) return false;
  L->part = 0;
  L->mom = align_up((size_t)n * sizeof(Partial));
  L->total = L->mom + align_up((size_t)n * sizeof(double));
  return true;
}

// Outcome-law workspace: the chain layout, then the residual masses and the
// per-(sequence, position) best weights and tokens.
struct OutcomeLayout {
  Layout L;
  size_t zk, lt, cw, cv, total;
};
bool outcome_layout(int B, int K, int V, int dtype, int n_top, OutcomeLayout* O) {
  if (n_top < 0 || n_top > SPEC_MAX_TOP) return false;
  if (!layout(B, K, V, dtype, 0, &O->L)) return false;
  const size_t slots = (size_t)B * (K + 1);
  O->zk = O->L.total;
  O->lt = O->zk + align_up(slots * sizeof(double));
  O->cw = O->lt + align_up((size_t)B * (2 * K + 1) * sizeof(double));
  O->cv = O->cw + align_up(slots * (size_t)n_top * sizeof(double));
  O->total = O->cv + align_up(slots * (size_t)n_top * sizeof(int));
  return true;
}

// Vocabulary-parallel workspace (one rank): the chain layout of the shard
// rows (partials, residual tile sums), then the per-sequence states and the
// prefixes of the tile sums.
struct VpLayout {
  Layout L;
  size_t seq, pre, total;
};
bool vp_layout(int B, int K, int Vs, int dtype, VpLayout* P) {
  if (!layout(B, K, Vs, dtype, 0, &P->L)) return false;
  P->seq = P->L.total;
  P->pre = P->seq + align_up((size_t)B * sizeof(VpSeq));
  P->total = P->pre + align_up((size_t)B * residual_tiles(Vs) * sizeof(double));
  return true;
}

bool rows_ok(const void* p, int64_t ld, int V, int dtype) {
  if (!p || !aligned(p, 16)) return false;
  if (ld < V) return false;
  return ((ld * elem_size(dtype)) % 16) == 0;
}

thread_local cudaError_t g_last_cuda = cudaSuccess;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SPEC_OK;
  g_last_cuda = e;
  return SPEC_ECUDA;
}

struct ChainCheck {
  Layout L;
  int rc;
};

ChainCheck check_chain(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                       int dtype, int B, int K, int V, const float* temperature, void* ws,
                       size_t ws_bytes) {
  ChainCheck c{};
  c.rc = SPEC_EINVAL;
  if (!layout(B, K, V, dtype, 0, &c.L)) return c;
  if (B == 0) { c.rc = SPEC_OK; return c; }
  if (!rows_ok(tgt, ld_tgt, V, dtype) || !temperature) return c;
  if (K > 0 && !rows_ok(drf, ld_drf, V, dtype)) return c;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < c.L.total) { c.rc = SPEC_EWORKSPACE; return c; }
  c.rc = SPEC_OK;
  return c;
}

RsBuffers rs_buffers(void* ws, const Layout& L) {
  RsBuffers b;
  b.part = reinterpret_cast<Partial*>((char*)ws + L.part);
  b.mom = nullptr;
  b.zero = nullptr;
  return b;
}

DecideCommon common_args(int dtype, int B, int K, int V, const int32_t* draft_tok,
                         const float* temperature, uint64_t seed, const int32_t* seq_id,
                         uint32_t round, double* diag, int32_t* dev_status, void* ws,
                         const Layout& L) {
  DecideCommon c;
  c.dtype = dtype;
  c.B = B;
  c.K = K;
  c.V = V;
  c.draft_tok = draft_tok;
  c.temperature = temperature;
  c.seed = seed;
  c.seq_id = seq_id;
  c.round = round;
  c.part = reinterpret_cast<const Partial*>((char*)ws + L.part);
  c.ntiles = stat_tiles(V, dtype);
  c.fin = reinterpret_cast<RowFinal*>((char*)ws + L.fin);
  c.diag = diag;
  c.status = dev_status;
  return c;
}

// Arguments of the verification step kernel for a chain call (workspace
// already checked).
StepArgs step_args(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                   int B, int K, int V, const int32_t* draft_tok, const float* temperature,
                   uint64_t seed, const int32_t* seq_id, uint32_t round, int32_t* accept_len,
                   int32_t* out_tok, double* diag, int32_t* dev_status, void* ws,
                   const Layout& L, int late_pos) {
  StepArgs a;
  std::memset(&a, 0, sizeof(a));
  const int es = elem_size(dtype);
  a.dtype = dtype;
  a.B = B;
  a.K = K;
  a.V = V;
  a.tgt = (const unsigned char*)tgt;
  a.drf = (const unsigned char*)drf;
  a.ld_tgt = ld_tgt * es;
  a.ld_drf = ld_drf * es;
  a.draft_tok = draft_tok;
  a.temperature = temperature;
  a.seed = seed;
  a.seq_id = seq_id;
  a.round = round;
  a.accept_len = accept_len;
  a.out_tok = out_tok;
  a.diag = diag;
  a.status = dev_status;
  a.nt = stat_tiles(V, dtype);
  a.NCe = (a.nt + kChunkTiles - 1) / kChunkTiles;
  a.NCl = (a.nt + kLateChunkTiles - 1) / kLateChunkTiles;
  a.NC = std::max(a.NCe, a.NCl);
  a.lp = std::min(late_pos, K);
  a.re = 2 * K + 1 - 2 * a.lp;
  a.rl = 2 * a.lp;
  a.n_early = (unsigned)((long long)B * a.re * a.NCe);
  a.n_total = a.n_early + (unsigned)((long long)B * a.rl * a.NCl);
  a.nrt = residual_tiles(V);
  a.D = (a.nrt + part_tiles(es) - 1) / part_tiles(es);
  char* w = (char*)ws;
  a.part = reinterpret_cast<ChunkStat*>(w + L.part);
  a.fin = reinterpret_cast<RowFinal*>(w + L.fin);
  a.seq = reinterpret_cast<SeqState*>(w + L.seq);
  a.tsum = reinterpret_cast<double*>(w + L.tsum);
  a.ptot = a.tsum + (size_t)B * a.nrt;
  a.ctr = reinterpret_cast<StepCounters*>(w + L.ctr);
  int* ints = reinterpret_cast<int*>(w + L.ints);
  a.seq_cnt = ints;
  a.seq_done = ints + B;
  a.draw_cnt = ints + 2 * B;
  a.tok_off = ints + 3 * B;
  a.tok_seq = ints + 4 * B;
  a.row_cnt = ints + (size_t)B * (4 + K + 1);
  return a;
}

}  // namespace

// The recorder behind every SPEC_ECUDA return of the library (other sources
// of the library return through it too, so spec_last_cuda_error names it).
int specv::record_cuda_status(cudaError_t e) { return cuda_status(e); }

// Host checks of a paged commit's arguments; fills *out. SPEC_OK with B == 0
// means nothing to do.
static int commit_args(int B, int block_size, int max_blocks, int32_t* block_tables,
                       int32_t* seq_lens, const int32_t* base_len, const int32_t* keep,
                       int keep_add, int32_t* free_stack, int32_t* free_top, int num_blocks,
                       int Kp1, const void* kv_stage, void* kv_pool, int layers, int kv_heads,
                       int head_dim, const void* hid_stage, void* hid_out, int32_t* hid_off,
                       int hidden, int32_t* dev_status, CommitArgs* out) {
  if (B < 0 || B > SPEC_MAX_COMMIT_B || block_size < 1 || max_blocks < 0 || num_blocks < 0 ||
      Kp1 < 0)
    return SPEC_EINVAL;
  if (B == 0) return SPEC_OK;
  if (!block_tables || !seq_lens || !keep || !free_stack || !free_top) return SPEC_EINVAL;
  if ((long long)B * Kp1 > (1LL << 31) - 1 || (long long)B * max_blocks > (1LL << 31) - 1)
    return SPEC_EINVAL;
  CommitArgs& a = *out;
  std::memset(&a, 0, sizeof(a));
  if ((kv_stage == nullptr) != (kv_pool == nullptr)) return SPEC_EINVAL;
  if (kv_stage) {
    if (layers < 1 || kv_heads < 1 || head_dim < 1) return SPEC_EINVAL;
    const long long seg = 2LL * kv_heads * head_dim;
    if (seg % 16 != 0 || seg > (1 << 30)) return SPEC_EINVAL;
    if (!aligned(kv_stage, 16) || !aligned(kv_pool, 16)) return SPEC_EINVAL;
    a.layers = layers;
    a.seg_bytes = (int)seg;
  }
  if ((hid_stage == nullptr) != (hid_out == nullptr)) return SPEC_EINVAL;
  if (hid_stage) {
    if (hidden < 1 || (2LL * hidden) % 16 != 0 || !hid_off) return SPEC_EINVAL;
    if (!aligned(hid_stage, 16) || !aligned(hid_out, 16)) return SPEC_EINVAL;
    a.hid_bytes = 2 * hidden;
  }
  a.B = B;
  a.block_size = block_size;
  a.max_blocks = max_blocks;
  a.num_blocks = num_blocks;
  a.Kp1 = Kp1;
  a.keep_add = keep_add;
  a.tables = block_tables;
  a.seq_lens = seq_lens;
  a.base_len = base_len;
  a.keep = keep;
  a.free_stack = free_stack;
  a.free_top = free_top;
  a.kv_stage = (const unsigned char*)kv_stage;
  a.kv_pool = (unsigned char*)kv_pool;
  a.hid_stage = (const unsigned char*)hid_stage;
  a.hid_out = (unsigned char*)hid_out;
  a.hid_off = hid_off;
  a.status = dev_status;
  return SPEC_OK;
}

#pragma GCC visibility push(default)
namespace {

struct VpCheck {
  VpLayout P;
  int rc;
};

VpCheck check_vp(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                 int B, int K, int Vs, int v0, int V, int R, int rank,
                 const int32_t* draft_tok, const float* temperature, void* ws,
                 size_t ws_bytes) {
  VpCheck c{};
  c.rc = SPEC_EINVAL;
  if (!vp_layout(B, K, Vs, dtype, &c.P)) return c;
  if (V < 1 || V > SPEC_MAX_V || v0 < 0 || v0 > V - Vs) return c;
  if (R < 1 || R > SPEC_VP_MAX_RANKS || rank < 0 || rank >= R) return c;
  if (B == 0) { c.rc = SPEC_OK; return c; }
  if (!rows_ok(tgt, ld_tgt, Vs, dtype) || !temperature) return c;
  if (K > 0 && (!rows_ok(drf, ld_drf, Vs, dtype) || !draft_tok)) return c;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < c.P.total) { c.rc = SPEC_EWORKSPACE; return c; }
  c.rc = SPEC_OK;
  return c;
}

VpArgs vp_args(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype, int B,
               int K, int Vs, int v0, int V, int R, int rank, const int32_t* draft_tok,
               const float* temperature, int32_t* dev_status, void* ws, const VpLayout& P) {
  VpArgs a{};
  const int es = elem_size(dtype);
  a.B = B;
  a.K = K;
  a.Vs = Vs;
  a.v0 = v0;
  a.V = V;
  a.R = R;
  a.rank = rank;
  a.tgt = (const unsigned char*)tgt;
  a.drf = (const unsigned char*)drf;
  a.ld_tgt = ld_tgt * es;
  a.ld_drf = ld_drf * es;
  a.draft_tok = draft_tok;
  a.temperature = temperature;
  a.part = reinterpret_cast<const Partial*>((char*)ws + P.L.part);
  a.ntiles = stat_tiles(Vs, dtype);
  a.seq = reinterpret_cast<VpSeq*>((char*)ws + P.seq);
  a.tsum = reinterpret_cast<double*>((char*)ws + P.L.tsum);
  a.pre = reinterpret_cast<double*>((char*)ws + P.pre);
  a.status = dev_status;
  return a;
}

}  // namespace

extern "C" {

size_t spec_workspace_bytes(int B, int K, int V, int dtype, int Ni) {
  Layout L;
  if (!layout(B, K, V, dtype, Ni, &L)) return 0;
  return L.total;
}

const char* spec_status_string(int status) {
  switch (status) {
    case SPEC_OK: return "ok";
    case SPEC_EINVAL: return "invalid argument or value";
    case SPEC_ECUDA: return "CUDA launch or API error";
    case SPEC_EWORKSPACE: return "workspace missing, misaligned or too small";
    case SPEC_ENOBLOCKS: return "free-block pool cannot cover the commit";
    case SPEC_ETIMEOUT: return "a bounded device wait ran out";
    case SPEC_EDEVICE: return "invalid input value found on the device";
    default: return "unknown status";
  }
}

// Leading positions whose rows the row-statistics kernel streams last, so
// the draw that follows finds them in L2: as many (at most cap) as fit in 60%
// of the L2 with rows_per_pos rows per position and sequence. At B=64, K=8,
// V=128256 bf16 one position measured best: the verify-and-commit step
// 82.4 us with one, 83.2 with two, 84.4 with three, 90.2 with none; the
// outcome law 155.9 us with one, 158.4 with two, 163.0 with three.
static int late_positions(int B, int V, int dtype, int rows_per_pos, int cap = 1) {
  static int l2s[kMaxDevs];  // bytes per device, looked up once per device (0: unknown)
  static bool known[kMaxDevs];
  const int dev = current_device();
  int l2 = 0;
  if (dev >= 0 && dev < kMaxDevs && known[dev]) {
    l2 = l2s[dev];
  } else {
    if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess) {
      cudaGetLastError();
      l2 = 0;
    }
    if (dev >= 0 && dev < kMaxDevs) {
      l2s[dev] = l2;
      known[dev] = true;
    }
  }
  const double per_pos = (double)B * rows_per_pos * V * elem_size(dtype);
  const int n = per_pos > 0.0 ? (int)(0.6 * l2 / per_pos) : 0;
  return n > cap ? cap : n;
}

int spec_chain_row_stats(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                         int dtype, int B, int K, int V, const float* temperature,
                         int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  const ChainCheck ck = check_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, ws,
                                    ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  const int es = elem_size(dtype);
  ChainRows rows;
  rows.tgt = (const unsigned char*)tgt;
  rows.drf = (const unsigned char*)drf;
  rows.ld_tgt = ld_tgt * es;
  rows.ld_drf = ld_drf * es;
  rows.temperature = temperature;
  rows.K = K;
  rows.late_pos = late_positions(B, V, dtype, 2);
  RsBuffers rb = rs_buffers(ws, ck.L);
  rb.zero = reinterpret_cast<int32_t*>((char*)ws + ck.L.ticket);  // for spec_chain_decide_commit
  return cuda_status(launch_row_stats(dtype, rows, B * (2 * K + 1), V, rb, dev_status,
                                      (cudaStream_t)stream));
}

// The check's launch arguments (spec_chain_decide, and the one-launch form
// of spec_verify_chain). small: launch the one-launch form.
static int chain_decide_call(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                             int dtype, int B, int K, int V, const int32_t* draft_tok,
                             const float* temperature, uint64_t seed, const int32_t* seq_id,
                             uint32_t round, int32_t* accept_len, int32_t* out_tok, double* diag,
                             int32_t* dev_status, void* ws, size_t ws_bytes, void* stream,
                             bool small) {
  const ChainCheck ck = check_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, ws,
                                    ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  if (!seq_id || !accept_len || !out_tok || (K > 0 && !draft_tok)) return SPEC_EINVAL;
  const int es = elem_size(dtype);
  ChainDecideArgs a;
  a.c = common_args(dtype, B, K, V, draft_tok, temperature, seed, seq_id, round, diag, dev_status,
                    ws, ck.L);
  a.tgt = (const unsigned char*)tgt;
  a.drf = (const unsigned char*)drf;
  a.ld_tgt = ld_tgt * es;
  a.ld_drf = ld_drf * es;
  a.accept_len = accept_len;
  a.out_tok = out_tok;
  return cuda_status(small ? launch_chain_small(a, (cudaStream_t)stream)
                           : launch_chain_decide(a, (cudaStream_t)stream));
}

int spec_chain_decide(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                      int B, int K, int V, const int32_t* draft_tok, const float* temperature,
                      uint64_t seed, const int32_t* seq_id, uint32_t round, int32_t* accept_len,
                      int32_t* out_tok, double* diag, int32_t* dev_status, void* ws,
                      size_t ws_bytes, void* stream) {
  return chain_decide_call(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok, temperature, seed,
                           seq_id, round, accept_len, out_tok, diag, dev_status, ws, ws_bytes,
                           stream, false);
}

int spec_verify_chain(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                      int B, int K, int V, const int32_t* draft_tok, const float* temperature,
                      uint64_t seed, const int32_t* seq_id, uint32_t round, int32_t* accept_len,
                      int32_t* out_tok, double* diag, int32_t* dev_status, void* ws,
                      size_t ws_bytes, void* stream) {
  if (!seq_id || !accept_len || !out_tok || (K > 0 && !draft_tok)) {
    Layout L;
    if (layout(B, K, V, dtype, 0, &L) && B == 0) return SPEC_OK;
    return SPEC_EINVAL;
  }
  if (V >= 1 && V <= SPEC_SMALL_V)
    return chain_decide_call(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok, temperature,
                             seed, seq_id, round, accept_len, out_tok, diag, dev_status, ws,
                             ws_bytes, stream, true);
  int rc = spec_chain_row_stats(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, dev_status,
                                ws, ws_bytes, stream);
  if (rc != SPEC_OK) return rc;
  return spec_chain_decide(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok, temperature, seed,
                           seq_id, round, accept_len, out_tok, diag, dev_status, ws, ws_bytes,
                           stream);
}

int spec_verify_chain_persistent(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                                 int dtype, int B, int K, int V, const int32_t* draft_tok,
                                 const float* temperature, uint64_t seed, const int32_t* seq_id,
                                 uint32_t round, int32_t* accept_len, int32_t* out_tok,
                                 double* diag, int32_t* dev_status, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (!seq_id || !accept_len || !out_tok || (K > 0 && !draft_tok)) {
    Layout L;
    if (layout(B, K, V, dtype, 0, &L) && B == 0) return SPEC_OK;
    return SPEC_EINVAL;
  }
  const ChainCheck ck = check_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, ws,
                                    ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  const StepArgs a = step_args(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok, temperature,
                               seed, seq_id, round, accept_len, out_tok, diag, dev_status, ws,
                               ck.L, late_positions(B, V, dtype, 2));
  return cuda_status(launch_chain_step(a, (cudaStream_t)stream));
}

int spec_verify_hier(const void* lg_d, const void* lg_i, const void* lg_f, int64_t ld, int dtype,
                     int B, int K, int V, int Ni, const int32_t* draft_tok,
                     const float* temperature, uint64_t seed, const int32_t* seq_id,
                     uint32_t round, int32_t* win_len, int32_t* win_tok, double* win_stat,
                     int32_t* acc1, int32_t* acc2, int32_t* commit_tok, int32_t* commit_n,
                     double* diag, int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  if (K < 1 || Ni < 1 || !layout(B, K, V, dtype, Ni, &L)) return SPEC_EINVAL;
  if (B == 0) return SPEC_OK;
  if (!rows_ok(lg_d, ld, V, dtype) || !rows_ok(lg_i, ld, V, dtype) || !rows_ok(lg_f, ld, V, dtype))
    return SPEC_EINVAL;
  if (!draft_tok || !temperature || !seq_id || !win_len || !win_tok || !win_stat || !acc1 ||
      !acc2 || !commit_tok || !commit_n)
    return SPEC_EINVAL;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < L.total) return SPEC_EWORKSPACE;
  const int es = elem_size(dtype);
  const int S = Ni + K + 1;
  cudaStream_t st = (cudaStream_t)stream;
  const RsBuffers rsb = rs_buffers(ws, L);

  HierDecideArgs a;
  a.c = common_args(dtype, B, K, V, draft_tok, temperature, seed, seq_id, round, diag, dev_status,
                    ws, L);
  a.lg_d = (const unsigned char*)lg_d;
  a.lg_i = (const unsigned char*)lg_i;
  a.lg_f = (const unsigned char*)lg_f;
  a.ld = ld * es;
  a.S = S;
  a.Ni = Ni;
  a.win_len = win_len;
  a.win_tok = win_tok;
  a.win_stat = win_stat;
  a.acc1 = acc1;
  a.acc2 = acc2;
  a.commit_tok = commit_tok;
  a.commit_n = commit_n;

  Hier1Rows r1;
  r1.lg_i = a.lg_i;
  r1.lg_d = a.lg_d;
  r1.ld = a.ld;
  r1.temperature = temperature;
  r1.win_len = win_len;
  r1.K = K;
  r1.S = S;
  r1.Ni = Ni;
  r1.late_pos = late_positions(B, V, dtype, 2);
  cudaError_t e = launch_row_stats(dtype, r1, B * (2 * K + 1), V, rsb, dev_status, st);
  if (e == cudaSuccess) e = launch_hier1_decide(a, st);
  Hier2Rows r2;
  r2.lg_f = a.lg_f;
  r2.ld = a.ld;
  r2.temperature = temperature;
  r2.win_len = win_len;
  r2.acc1 = acc1;
  r2.S = S;
  r2.Ni = Ni;
  r2.late_pos = late_positions(B, V, dtype, 1);
  if (e == cudaSuccess) e = launch_row_stats(dtype, r2, B * S, V, rsb, dev_status, st);
  if (e == cudaSuccess) e = launch_hier2_decide(a, st);
  return cuda_status(e);
}

int spec_commit_paged(int B, int block_size, int max_blocks, int32_t* block_tables,
                      int32_t* seq_lens, const int32_t* base_len, const int32_t* keep, int keep_add,
                      int32_t* free_stack, int32_t* free_top, int num_blocks, int Kp1,
                      const void* kv_stage, void* kv_pool, int layers, int kv_heads, int head_dim,
                      const void* hid_stage, void* hid_out, int32_t* hid_off, int hidden,
                      int32_t* dev_status, void* stream) {
  CommitArgs a;
  const int rc = commit_args(B, block_size, max_blocks, block_tables, seq_lens, base_len, keep,
                             keep_add, free_stack, free_top, num_blocks, Kp1, kv_stage, kv_pool,
                             layers, kv_heads, head_dim, hid_stage, hid_out, hid_off, hidden,
                             dev_status, &a);
  if (rc != SPEC_OK || B == 0) return rc;
  return cuda_status(launch_commit(a, (cudaStream_t)stream));
}

int spec_chain_decide_commit(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                             int dtype, int B, int K, int V, const int32_t* draft_tok,
                             const float* temperature, uint64_t seed, const int32_t* seq_id,
                             uint32_t round, int32_t* accept_len, int32_t* out_tok, double* diag,
                             int block_size, int max_blocks, int32_t* block_tables,
                             int32_t* seq_lens, const int32_t* base_len, int32_t* free_stack,
                             int32_t* free_top, int num_blocks, const void* kv_stage,
                             void* kv_pool, int layers, int kv_heads, int head_dim,
                             const void* hid_stage, void* hid_out, int32_t* hid_off, int hidden,
                             int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  if (B < 0 || B > SPEC_MAX_FUSED_B || K < 0 || K > SPEC_MAX_K) return SPEC_EINVAL;
  FusedArgs f;
  const int rc = commit_args(B, block_size, max_blocks, block_tables, seq_lens, base_len,
                             accept_len, 1, free_stack, free_top, num_blocks, K + 1, kv_stage,
                             kv_pool, layers, kv_heads, head_dim, hid_stage, hid_out, hid_off,
                             hidden, dev_status, &f.cm);
  if (rc != SPEC_OK) return rc;
  const ChainCheck ck = check_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, ws,
                                    ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  if (!seq_id || !out_tok || (K > 0 && !draft_tok)) return SPEC_EINVAL;
  const int es = elem_size(dtype);
  f.d.c = common_args(dtype, B, K, V, draft_tok, temperature, seed, seq_id, round, diag,
                      dev_status, ws, ck.L);
  f.d.tgt = (const unsigned char*)tgt;
  f.d.drf = (const unsigned char*)drf;
  f.d.ld_tgt = ld_tgt * es;
  f.d.ld_drf = ld_drf * es;
  f.d.accept_len = accept_len;
  f.d.out_tok = out_tok;
  f.ticket = reinterpret_cast<int32_t*>((char*)ws + ck.L.ticket);
  f.plan_flag = f.ticket + 32;  // its own 128-byte line: the leaders' ticket atomics stay apart
  f.rec = reinterpret_cast<CommitRec*>((char*)ws + ck.L.rec);
  return cuda_status(launch_chain_fused(f, (cudaStream_t)stream));
}

int spec_verify_chain_commit(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                             int dtype, int B, int K, int V, const int32_t* draft_tok,
                             const float* temperature, uint64_t seed, const int32_t* seq_id,
                             uint32_t round, int32_t* accept_len, int32_t* out_tok, double* diag,
                             int block_size, int max_blocks, int32_t* block_tables,
                             int32_t* seq_lens, const int32_t* base_len, int32_t* free_stack,
                             int32_t* free_top, int num_blocks, const void* kv_stage,
                             void* kv_pool, int layers, int kv_heads, int head_dim,
                             const void* hid_stage, void* hid_out, int32_t* hid_off, int hidden,
                             int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  // Every host check of the second half first, so a refused call launches nothing.
  if (B < 0 || B > SPEC_MAX_FUSED_B || K < 0 || K > SPEC_MAX_K) return SPEC_EINVAL;
  CommitArgs cm;
  int rc = commit_args(B, block_size, max_blocks, block_tables, seq_lens, base_len, accept_len,
                       1, free_stack, free_top, num_blocks, K + 1, kv_stage, kv_pool, layers,
                       kv_heads, head_dim, hid_stage, hid_out, hid_off, hidden, dev_status, &cm);
  if (rc != SPEC_OK) return rc;
  const ChainCheck ck = check_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, ws,
                                    ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  if (!seq_id || !out_tok || (K > 0 && !draft_tok)) return SPEC_EINVAL;
  rc = spec_chain_row_stats(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, dev_status,
                            ws, ws_bytes, stream);
  if (rc != SPEC_OK) return rc;
  return spec_chain_decide_commit(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok,
                                  temperature, seed, seq_id, round, accept_len, out_tok, diag,
                                  block_size, max_blocks, block_tables, seq_lens, base_len,
                                  free_stack, free_top, num_blocks, kv_stage, kv_pool, layers,
                                  kv_heads, head_dim, hid_stage, hid_out, hid_off, hidden,
                                  dev_status, ws, ws_bytes, stream);
}

int spec_verify_chain_commit_persistent(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                             int dtype, int B, int K, int V, const int32_t* draft_tok,
                             const float* temperature, uint64_t seed, const int32_t* seq_id,
                             uint32_t round, int32_t* accept_len, int32_t* out_tok, double* diag,
                             int block_size, int max_blocks, int32_t* block_tables,
                             int32_t* seq_lens, const int32_t* base_len, int32_t* free_stack,
                             int32_t* free_top, int num_blocks, const void* kv_stage,
                             void* kv_pool, int layers, int kv_heads, int head_dim,
                             const void* hid_stage, void* hid_out, int32_t* hid_off, int hidden,
                             int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  // Every host check of the second half first, so a refused call launches nothing.
  if (B < 0 || B > SPEC_MAX_FUSED_B || K < 0 || K > SPEC_MAX_K) return SPEC_EINVAL;
  CommitArgs cm;
  int rc = commit_args(B, block_size, max_blocks, block_tables, seq_lens, base_len, accept_len,
                       1, free_stack, free_top, num_blocks, K + 1, kv_stage, kv_pool, layers,
                       kv_heads, head_dim, hid_stage, hid_out, hid_off, hidden, dev_status, &cm);
  if (rc != SPEC_OK) return rc;
  const ChainCheck ck = check_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, temperature, ws,
                                    ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  if (!seq_id || !out_tok || (K > 0 && !draft_tok)) return SPEC_EINVAL;
  StepArgs a = step_args(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok, temperature, seed,
                         seq_id, round, accept_len, out_tok, diag, dev_status, ws, ck.L,
                         late_positions(B, V, dtype, 2));
  a.commit = 1;
  a.cm = cm;
  if (cm.kv_stage) {
    const int nseg = cm.layers * 2;
    a.unit_segs = std::max(1, kCopyUnit / cm.seg_bytes);
    a.units_kv = (nseg + a.unit_segs - 1) / a.unit_segs;
  }
  a.units_tok = a.units_kv + (cm.hid_stage ? 1 : 0);
  return cuda_status(launch_chain_step(a, (cudaStream_t)stream));
}

size_t spec_draft_workspace_bytes(int B, int V, int dtype) {
  DraftLayout L;
  if (!draft_layout(B, V, dtype, &L)) return 0;
  return L.total;
}

int spec_draft_sample(const void* logits, int64_t ld, int dtype, int B, int V,
                      const float* temperature, uint64_t seed, const int32_t* seq_id,
                      uint32_t round, const int32_t* pos, int32_t* out_tok, double* out_logq,
                      double* out_entropy, int32_t* dev_status, void* ws, size_t ws_bytes,
                      void* stream) {
  DraftLayout L;
  if (!draft_layout(B, V, dtype, &L)) return SPEC_EINVAL;
  if (B == 0) return SPEC_OK;
  if (!rows_ok(logits, ld, V, dtype) || !temperature || !seq_id || !pos || !out_tok)
    return SPEC_EINVAL;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < L.total) return SPEC_EWORKSPACE;
  return cuda_status(launch_draft_step(
      dtype, (const unsigned char*)logits, ld * elem_size(dtype), B, V, temperature, seed, seq_id,
      round, pos, reinterpret_cast<Partial*>((char*)ws + L.part),
      reinterpret_cast<double*>((char*)ws + L.mom), out_tok, out_logq, out_entropy, dev_status,
      (cudaStream_t)stream));
}

size_t spec_outcome_workspace_bytes(int B, int K, int V, int dtype, int n_top) {
  OutcomeLayout O;
  if (!outcome_layout(B, K, V, dtype, n_top, &O)) return 0;
  return O.total;
}

int spec_outcome_law(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                     int B, int K, int V, const int32_t* draft_tok, const float* temperature,
                     int n_top, double* p_len, double* beta, double* mass, int32_t* top_len,
                     int32_t* top_tok, double* top_prob, int32_t* dev_status, void* ws,
                     size_t ws_bytes, void* stream) {
  OutcomeLayout O;
  if (!outcome_layout(B, K, V, dtype, n_top, &O)) return SPEC_EINVAL;
  if (B == 0) return SPEC_OK;
  if (!rows_ok(tgt, ld_tgt, V, dtype) || !temperature || !p_len) return SPEC_EINVAL;
  if (K > 0 && (!rows_ok(drf, ld_drf, V, dtype) || !draft_tok)) return SPEC_EINVAL;
  if (n_top > 0 && (!top_len || !top_tok || !top_prob)) return SPEC_EINVAL;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < O.total) return SPEC_EWORKSPACE;
  const int es = elem_size(dtype);
  ChainRows rows;
  rows.tgt = (const unsigned char*)tgt;
  rows.drf = (const unsigned char*)drf;
  rows.ld_tgt = ld_tgt * es;
  rows.ld_drf = ld_drf * es;
  rows.temperature = temperature;
  rows.K = K;
  // every row pair is read again: those of the first late_pos positions are
  // streamed last, to be still in L2 when the pair pass reads them
  rows.late_pos = late_positions(B, V, dtype, 2);
  const cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = launch_row_stats(dtype, rows, B * (2 * K + 1), V, rs_buffers(ws, O.L),
                                   dev_status, st);
  if (e != cudaSuccess) return cuda_status(e);
  OutcomeArgs a;
  a.B = B;
  a.K = K;
  a.V = V;
  a.n_top = n_top;
  a.ntiles = stat_tiles(V, dtype);
  a.tgt = rows.tgt;
  a.drf = rows.drf;
  a.ld_tgt = rows.ld_tgt;
  a.ld_drf = rows.ld_drf;
  a.draft_tok = draft_tok;
  a.temperature = temperature;
  a.part = reinterpret_cast<const Partial*>((char*)ws + O.L.part);
  a.zk = reinterpret_cast<double*>((char*)ws + O.zk);
  a.lt = reinterpret_cast<double*>((char*)ws + O.lt);
  a.cw = reinterpret_cast<double*>((char*)ws + O.cw);
  a.late_pos = rows.late_pos;
  a.cv = reinterpret_cast<int*>((char*)ws + O.cv);
  a.p_len = p_len;
  a.beta = beta;
  a.mass = mass;
  a.top_len = top_len;
  a.top_tok = top_tok;
  a.top_prob = top_prob;
  a.status = dev_status;
  return cuda_status(launch_outcome(dtype, a, st));
}

int spec_saguaro_adjust(void* logits, int64_t ld, int dtype, int B, int rows_per_seq, int V,
                        const int32_t* cached, int n_cached, int per_row, double eps,
                        const float* temperature, void* stream) {
  if (B < 0 || rows_per_seq < 0 || V < 1 || V > SPEC_MAX_V || n_cached < 0 ||
      n_cached > SPEC_MAX_CACHED || (per_row != 0 && per_row != 1))
    return SPEC_EINVAL;
  if (dtype != SPEC_F32 && dtype != SPEC_BF16) return SPEC_EINVAL;
  if (!(eps >= 0.0 && eps < 1.0)) return SPEC_EINVAL;
  if (B == 0 || n_cached == 0 || rows_per_seq == 0 || eps == 0.0) return SPEC_OK;
  if (!logits || ld < V || !cached || !temperature) return SPEC_EINVAL;
  return cuda_status(launch_saguaro_adjust(
      dtype, (unsigned char*)logits, ld * elem_size(dtype), B, rows_per_seq, V, cached, n_cached,
      per_row, std::log1p(-eps), temperature, (cudaStream_t)stream));
}

// ---------------------------------------------------------------------------
// Vocabulary-parallel chain verification
// ---------------------------------------------------------------------------
size_t spec_vp_workspace_bytes(int B, int K, int Vs, int dtype) {
  VpLayout P;
  if (!vp_layout(B, K, Vs, dtype, &P)) return 0;
  return P.total;
}

int spec_vp_shard_stats(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                        int dtype, int B, int K, int Vs, int v0, int V,
                        const int32_t* draft_tok, const float* temperature, void* rows_out,
                        int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  const VpCheck ck = check_vp(tgt, ld_tgt, drf, ld_drf, dtype, B, K, Vs, v0, V, 1, 0, draft_tok,
                              temperature, ws, ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  if (!rows_out || !aligned(rows_out, 8)) return SPEC_EINVAL;
  const cudaStream_t st = (cudaStream_t)stream;
  ChainRows rows;
  rows.tgt = (const unsigned char*)tgt;
  rows.drf = (const unsigned char*)drf;
  rows.ld_tgt = ld_tgt * elem_size(dtype);
  rows.ld_drf = ld_drf * elem_size(dtype);
  rows.temperature = temperature;
  rows.K = K;
  rows.late_pos = 0;
  const RsBuffers rb = rs_buffers(ws, ck.P.L);
  cudaError_t e = launch_row_stats(dtype, rows, B * (2 * K + 1), Vs, rb, dev_status, st);
  if (e != cudaSuccess) return cuda_status(e);
  VpArgs a = vp_args(tgt, ld_tgt, drf, ld_drf, dtype, B, K, Vs, v0, V, 1, 0, draft_tok,
                     temperature, dev_status, ws, ck.P);
  a.rows = reinterpret_cast<VpRow*>(rows_out);
  return cuda_status(launch_vp_records(dtype, a, st));
}

int spec_vp_decide(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                   int B, int K, int Vs, int v0, int V, int R, int rank, const void* rows_all,
                   const int32_t* draft_tok, const float* temperature, uint64_t seed,
                   const int32_t* seq_id, uint32_t round, void* mass_out, double* diag,
                   int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  const VpCheck ck = check_vp(tgt, ld_tgt, drf, ld_drf, dtype, B, K, Vs, v0, V, R, rank,
                              draft_tok, temperature, ws, ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  if (!rows_all || !aligned(rows_all, 8) || !mass_out || !aligned(mass_out, 8) || !seq_id)
    return SPEC_EINVAL;
  VpArgs a = vp_args(tgt, ld_tgt, drf, ld_drf, dtype, B, K, Vs, v0, V, R, rank, draft_tok,
                     temperature, dev_status, ws, ck.P);
  a.rows_all = reinterpret_cast<const VpRow*>(rows_all);
  a.mass = reinterpret_cast<VpMass*>(mass_out);
  a.seed = seed;
  a.seq_id = seq_id;
  a.round = round;
  a.diag = diag;
  return cuda_status(launch_vp_decide(dtype, a, (cudaStream_t)stream));
}

int spec_vp_pick(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf, int dtype,
                 int B, int K, int Vs, int v0, int V, int R, int rank, const void* mass_all,
                 const int32_t* draft_tok, const float* temperature, int32_t* accept_len,
                 int32_t* out_tok, double* diag, int32_t* dev_status, void* ws, size_t ws_bytes,
                 void* stream) {
  const VpCheck ck = check_vp(tgt, ld_tgt, drf, ld_drf, dtype, B, K, Vs, v0, V, R, rank,
                              draft_tok, temperature, ws, ws_bytes);
  if (ck.rc != SPEC_OK || B == 0) return ck.rc;
  if (!mass_all || !aligned(mass_all, 8) || !accept_len || !out_tok) return SPEC_EINVAL;
  VpArgs a = vp_args(tgt, ld_tgt, drf, ld_drf, dtype, B, K, Vs, v0, V, R, rank, draft_tok,
                     temperature, dev_status, ws, ck.P);
  a.mass_all = reinterpret_cast<const VpMass*>(mass_all);
  a.accept_len = accept_len;
  a.out_tok = out_tok;
  a.diag = diag;
  return cuda_status(launch_vp_pick(dtype, a, (cudaStream_t)stream));
}

const char* spec_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

int spec_philox_uniforms(uint64_t seed, const uint32_t* ctr, int n, float* out, void* stream) {
  if (n < 0 || (n > 0 && (!ctr || !out))) return SPEC_EINVAL;
  return cuda_status(launch_philox(seed, ctr, n, out, (cudaStream_t)stream));
}

}  // extern "C"
#pragma GCC visibility pop
