// sv_api.cu -- the C ABI of libspecverify.so (include/spec_verify.h):
// argument validation, chunk planning, workspace layout and kernel dispatch.
// Host code only; every step of the verify path runs in sv_kernels.cu.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <utility>

#include "spec_verify.h"
#include "sv_internal.h"

namespace sv {

Plan plan_chunks(long long rows, int V, int bpe, int es_min, int chunk_bytes) {
  const int ch = full_chunk_entries(chunk_bytes < kStageBytes ? chunk_bytes : kStageBytes, bpe,
                                    es_min);
  long long nch = (V + ch - 1) / ch;
  // Small calls: split rows finer (chunks of >= 512 entries) so that about
  // 2048 chunks spread over the SMs.
  const long long want = 2048;
  if (rows > 0 && rows * nch < want) {
    const long long finer = (want + rows - 1) / rows;
    const long long most = (V + 511) / 512;
    const long long n2 = finer < most ? finer : most;
    if (n2 > nch) {
      long long c = (V + n2 - 1) / n2;
      c = (c + 7) / 8 * 8;
      return Plan{static_cast<int>(c), static_cast<int>((V + c - 1) / c)};
    }
  }
  return Plan{ch, static_cast<int>(nch)};
}

namespace {

constexpr size_t kCtrlBytes = sizeof(Ctrl);

int elem_bytes(int dtype) { return dtype == SV_BF16 ? 2 : 4; }
bool dtype_ok(int dtype) { return dtype == SV_F32 || dtype == SV_BF16; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool stride16(long long stride, int es) { return ((stride * es) % 16) == 0; }

size_t seq_bytes(int B) { return static_cast<size_t>(B) * sizeof(SeqRec); }

// Elements a strided view spans: one past its last element.
long long span(std::initializer_list<std::pair<long long, long long>> dims, int V) {
  long long last = V - 1;
  for (const auto& d : dims) last += (d.first - 1) * d.second;  // (extent, stride)
  return last + 1;
}

// Partial slots (8 bytes each) and row counters (4 bytes each):
//   stochastic: chunk [B][k][nch][2], row [B][k][2], phase-2 [B][nch],
//               ready list [B], rc [B][k]
//   argmax:     chunk [B][R][nch], row [B][R], rc [B][R], branch state [rows]
//               (R = G (k+1))
struct StochLayout {
  size_t p1, r1, p2, list, rc, bytes;  // offsets from the tail, in bytes
};
StochLayout stochastic_layout(int B, int k, int nch) {
  StochLayout l;
  const size_t bk = static_cast<size_t>(B) * k;
  l.p1 = 0;
  l.r1 = l.p1 + bk * nch * 2 * 8;
  l.p2 = l.r1 + bk * 2 * 8;
  l.list = l.p2 + static_cast<size_t>(B) * nch * 8;
  l.rc = l.list + static_cast<size_t>(B) * 8;
  l.bytes = l.rc + (bk * 4 + 15) / 16 * 16;
  return l;
}
struct ArgLayout {
  size_t slots, rkey, rc, dead, bytes;
};
// dead holds one word per (sequence, branch); `rows` words bound it in
// every mode.
ArgLayout argmax_layout(long long rows, int nch) {
  ArgLayout l;
  l.slots = 0;
  l.rkey = static_cast<size_t>(rows) * nch * 8;
  l.rc = l.rkey + static_cast<size_t>(rows) * 8;
  l.dead = l.rc + (static_cast<size_t>(rows) * 4 + 15) / 16 * 16;
  l.bytes = l.dead + (static_cast<size_t>(rows) * 4 + 15) / 16 * 16;
  return l;
}

size_t stochastic_part_bytes(int B, int k, int V, int bpe, int es_min) {
  const Plan pl = plan_chunks(static_cast<long long>(B) * k, V, bpe, es_min, kStochChunkBytes);
  return stochastic_layout(B, k, pl.nch).bytes;
}

// Threshold acceptance: the argmax layout followed by chunk statistics
// [B][k+1][nch] and row statistics [B][k+1] (8 bytes each).
struct ThreshLayout {
  ArgLayout a;
  size_t sslots, rstats, bytes;
};
ThreshLayout threshold_layout(long long rows, int nch) {
  ThreshLayout l;
  l.a = argmax_layout(rows, nch);
  l.sslots = l.a.bytes;
  l.rstats = l.sslots + static_cast<size_t>(rows) * nch * 8;
  l.bytes = l.rstats + static_cast<size_t>(rows) * 8;
  return l;
}

size_t argmax_key_bytes(int B, int G, int k, int V, int es) {
  const long long rows = static_cast<long long>(B) * G * (k + 1);
  return argmax_layout(rows, plan_chunks(rows, V, es, es, kArgmaxChunkBytes).nch).bytes;
}

bool sizes_ok(int B, int G, int k, int V) {
  return B >= 0 && G >= 1 && G <= 64 && k >= 0 && k <= 32 && V >= 1;
}

int sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

struct WsView {
  Ctrl* ctrl;
  SeqRec* seq;
  void* tail;
};

// Plain greedy / multi-candidate calls whose logits take at most this many
// bytes run as one grid of row-chunk blocks instead of the persistent
// pipeline (the pipeline's ramp and tail, and early exit's need for a
// rejection to be known a whole position block ahead, only pay off on larger
// calls).  SV_ONESHOT_MAX_BYTES overrides it (0: never), for tests and tuning.
// Measured on B200 (one grid vs the pipeline, µs per call in a graph of
// calls on four copies of the logits): greedy, k = 4, V = 128256: B = 16
// (20.5 MB) 11.6 vs 22.2, 64 19.8 vs 28.1, 128 30.2 vs 40.1, 256 (328 MB)
// 52.6 vs 58.4, 512 (657 MB) 95.6 vs 92.3, 1024 183.5 vs 168.2;
// multi-candidate, G = 8, k = 4, V = 32000: B = 16 15.9 vs 33.2, 64 33.6 vs
// 51.2, 256 (655 MB) 97.7 vs 122.7.
constexpr long long kOneshotMaxBytes = 512ll << 20;

// Stochastic calls of at least this many sequences park phase-1 chunks of
// pairs whose earlier rows are undecided; parking measured faster at every
// batch size tried (1, 64, 256), so by default every call does.
// SV_PARK_MIN_B overrides it (the GPU tests run both ways).
#ifndef SV_PARK_MIN_B_DEFAULT
#define SV_PARK_MIN_B_DEFAULT 1
#endif
bool park_tickets(int B) {
  long long limit = SV_PARK_MIN_B_DEFAULT;
  if (const char* env = std::getenv("SV_PARK_MIN_B")) limit = std::atoll(env);
  return B >= limit;
}

bool use_oneshot(long long bytes) {
  long long limit = kOneshotMaxBytes;
  if (const char* env = std::getenv("SV_ONESHOT_MAX_BYTES")) limit = std::atoll(env);
  return bytes <= limit;
}

WsView carve(void* ws, int B) {
  unsigned char* base = static_cast<unsigned char*>(ws);
  return WsView{reinterpret_cast<Ctrl*>(base), reinterpret_cast<SeqRec*>(base + kCtrlBytes),
                base + kCtrlBytes + seq_bytes(B)};
}

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" size_t spec_verify_workspace_size(int B, int G, int k, int V) {
  if (!sizes_ok(B, G, k, V)) return 0;
  size_t tail = 0;
  for (int es : {2, 4}) {
    const size_t a = argmax_key_bytes(B, G, k, V, es);
    if (a > tail) tail = a;
  }
  if (G == 1) {
    for (int es : {2, 4}) {  // threshold acceptance
      const long long rows = static_cast<long long>(B) * (k + 1);
      const size_t t =
          threshold_layout(rows, plan_chunks(rows, V, es, es, kArgmaxChunkBytes).nch).bytes;
      if (t > tail) tail = t;
    }
    // (bytes per entry, narrowest element) of bf16/bf16, bf16/fp32 (either
    // way round) and fp32/fp32 pairs
    static const int kPairs[3][2] = {{4, 2}, {6, 2}, {8, 4}};
    for (const auto& pr : kPairs) {
      const size_t s = stochastic_part_bytes(B, k, V, pr[0], pr[1]);
      if (s > tail) tail = s;
    }
  }
  const size_t total = kCtrlBytes + seq_bytes(B) + tail;
  return (total + 255) / 256 * 256;
}

namespace sv {
namespace {
std::atomic<unsigned long long> g_launches{0};
}  // namespace
cudaError_t counted(cudaError_t e, int n) {
  if (e == cudaSuccess) g_launches.fetch_add(static_cast<unsigned long long>(n));
  return e;
}
unsigned long long launches_so_far() { return g_launches.load(); }
}  // namespace sv

extern "C" unsigned long long spec_verify_kernel_launches(void) { return sv::launches_so_far(); }

extern "C" const char* spec_verify_status_string(int status) {
  switch (status) {
    case SV_OK: return "SV_OK";
    case SV_ERR_INVALID_ARG: return "SV_ERR_INVALID_ARG: invalid argument";
    case SV_ERR_MISALIGNED: return "SV_ERR_MISALIGNED: pointer not aligned";
    case SV_ERR_WORKSPACE: return "SV_ERR_WORKSPACE: workspace too small";
    case SV_ERR_CUDA: return "SV_ERR_CUDA: CUDA runtime error";
    case SV_ERR_DEVICE_TIMEOUT: return "SV_ERR_DEVICE_TIMEOUT: a device wait timed out";
    default: return "unknown spec_verify status";
  }
}

extern "C" int spec_verify_workspace_init(void* workspace, size_t workspace_bytes,
                                          void* stream) {
  if (!workspace) return SV_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return SV_ERR_MISALIGNED;
  if (cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SV_ERR_CUDA;
  return SV_OK;
}

extern "C" int spec_verify_read_device_status(void* workspace, uint32_t* flags_host, int clear,
                                              void* stream) {
  if (!workspace || !flags_host) return SV_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return SV_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ctrl* ctrl = static_cast<Ctrl*>(workspace);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, &ctrl->flags, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SV_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SV_ERR_CUDA;
  *flags_host = v;
  if (clear && cudaMemsetAsync(&ctrl->flags, 0, sizeof v, st) != cudaSuccess) return SV_ERR_CUDA;
  return SV_OK;
}

extern "C" int spec_verify_stochastic(const void* target_logits, int t_dtype,
                                      int64_t t_stride_b, int64_t t_stride_pos,
                                      const void* draft_logits, int d_dtype, int64_t d_stride_b,
                                      int64_t d_stride_pos, const int32_t* draft_tokens, int B,
                                      int k, int V, float temperature, uint64_t seed,
                                      uint32_t seq_offset, int32_t* accepted_len,
                                      int32_t* out_tokens, float* probs_out, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!sizes_ok(B, 1, k, V)) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!target_logits || !accepted_len || !out_tokens || !workspace) return SV_ERR_INVALID_ARG;
  if (k > 0 && (!draft_logits || !draft_tokens)) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(t_dtype) || !dtype_ok(d_dtype)) return SV_ERR_INVALID_ARG;
  if (!(temperature > 0.0f) || !std::isfinite(temperature) || !std::isnormal(temperature))
    return SV_ERR_INVALID_ARG;
  if (t_stride_b < 0 || t_stride_pos < 0 || d_stride_b < 0 || d_stride_pos < 0)
    return SV_ERR_INVALID_ARG;
  const int st = elem_bytes(t_dtype), sd = elem_bytes(d_dtype);
  if (!aligned(target_logits, st) || (k > 0 && !aligned(draft_logits, sd)) ||
      !aligned(accepted_len, 4) || !aligned(out_tokens, 4) ||
      (k > 0 && !aligned(draft_tokens, 4)) || (probs_out && !aligned(probs_out, 4)) ||
      !aligned(workspace, 16))
    return SV_ERR_MISALIGNED;
  if (workspace_bytes < spec_verify_workspace_size(B, 1, k, V)) return SV_ERR_WORKSPACE;

  const int grid = sm_count();
  if (grid <= 0) return SV_ERR_CUDA;
  const Plan pl = plan_chunks(static_cast<long long>(B) * k, V, st + sd, st < sd ? st : sd, kStochChunkBytes);
  const long long total1 = static_cast<long long>(k) * B * pl.nch;
  const long long total2 = static_cast<long long>(B) * pl.nch;
  if (total1 + total2 >= (1ll << 31)) return SV_ERR_INVALID_ARG;

  const bool tma = aligned(target_logits, 16) && stride16(t_stride_b, st) &&
                   stride16(t_stride_pos, st) &&
                   (k == 0 || (aligned(draft_logits, 16) && stride16(d_stride_b, sd) &&
                               stride16(d_stride_pos, sd)));

  const WsView ws = carve(workspace, B);
  StochParams p{};
  p.tgt = target_logits;
  p.t_sb = t_stride_b;
  p.t_sp = t_stride_pos;
  p.drf = draft_logits;
  p.d_sb = d_stride_b;
  p.d_sp = d_stride_pos;
  p.t_elems = span({{B, t_stride_b}, {k + 1, t_stride_pos}}, V);
  p.d_elems = k > 0 ? span({{B, d_stride_b}, {k, d_stride_pos}}, V) : 0;
  p.tokens = draft_tokens;
  p.B = B;
  p.k = k;
  p.V = V;
  p.c2 = 1.4426950408889634f / temperature;
  p.key0 = static_cast<unsigned int>(seed & 0xffffffffull);
  p.key1 = static_cast<unsigned int>(seed >> 32);
  p.seq_offset = seq_offset;
  p.accepted_len = accepted_len;
  p.out_tokens = out_tokens;
  p.probs = probs_out;
  p.ch = pl.ch;
  p.nch = pl.nch;
  p.total1 = static_cast<unsigned int>(total1);
  p.total2 = static_cast<unsigned int>(total2);
  p.park = park_tickets(B) ? 1 : 0;
  p.div_nch = make_udiv(static_cast<unsigned int>(pl.nch));
  p.div_B = make_udiv(static_cast<unsigned int>(B));
  p.ctrl = ws.ctrl;
  p.seq = ws.seq;
  const StochLayout lay = stochastic_layout(B, k, pl.nch);
  unsigned char* tail = static_cast<unsigned char*>(ws.tail);
  p.p1 = reinterpret_cast<unsigned long long*>(tail + lay.p1);
  p.r1 = reinterpret_cast<unsigned long long*>(tail + lay.r1);
  p.p2 = reinterpret_cast<unsigned long long*>(tail + lay.p2);
  p.rc = reinterpret_cast<unsigned int*>(tail + lay.rc);
  p.list = reinterpret_cast<unsigned long long*>(tail + lay.list);
  const cudaError_t e = launch_stochastic(p, t_dtype, d_dtype, tma, grid, kernel_smem_bytes(),
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

// R == 0: rows g*(k+1)+i of a [B, G, k+1, V] tensor; R > 0: R rows per
// sequence at stride sg, either the rows form (row_of maps (b, g, i) to a
// row) or a tree of R = k + 1 nodes (parent pointers, G = 1, path out).
static int argmax_call(const void* target_logits, int t_dtype, int64_t sb, int64_t sg,
                       int64_t sp, const int32_t* tokens, int B, int G, int k, int V, int R,
                       const int32_t* row_of, const int32_t* parent, int32_t* path,
                       int32_t* best_g, int32_t* accepted_len, int32_t* out_tokens,
                       void* workspace, size_t workspace_bytes, void* stream,
                       size_t need_bytes, float temperature = 0.0f, float threshold = 0.0f) {
  const bool thresh = threshold > 0.0f;
  if (!sizes_ok(B, G, k, V)) return SV_ERR_INVALID_ARG;
  const long long full_rows = static_cast<long long>(G) * (k + 1);
  if (R < 0 || R > full_rows || (R > 0) != (row_of != nullptr || parent != nullptr) ||
      (row_of && parent))
    return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (parent && !path) return SV_ERR_INVALID_ARG;
  if (!target_logits || !accepted_len || !out_tokens || !workspace) return SV_ERR_INVALID_ARG;
  if (k > 0 && !tokens) return SV_ERR_INVALID_ARG;
  if (!dtype_ok(t_dtype)) return SV_ERR_INVALID_ARG;
  if (sb < 0 || sg < 0 || sp < 0) return SV_ERR_INVALID_ARG;
  const int st = elem_bytes(t_dtype);
  if (!aligned(target_logits, st) || !aligned(accepted_len, 4) || !aligned(out_tokens, 4) ||
      (k > 0 && !aligned(tokens, 4)) || (best_g && !aligned(best_g, 4)) ||
      (row_of && !aligned(row_of, 4)) || (parent && !aligned(parent, 4)) ||
      (path && !aligned(path, 4)) || !aligned(workspace, 16))
    return SV_ERR_MISALIGNED;
  if (workspace_bytes < need_bytes) return SV_ERR_WORKSPACE;

  const int grid = sm_count();
  if (grid <= 0) return SV_ERR_CUDA;
  const int rows_per_seq = R > 0 ? R : static_cast<int>(full_rows);
  const long long rows = static_cast<long long>(B) * rows_per_seq;
  const Plan pl = plan_chunks(rows, V, st, st, kArgmaxChunkBytes);
  const long long total = rows * pl.nch;
  if (total >= (1ll << 31)) return SV_ERR_INVALID_ARG;
  const bool tma = aligned(target_logits, 16) && stride16(sb, st) && stride16(sg, st) &&
                   (R > 0 || stride16(sp, st));

  const WsView ws = carve(workspace, B);
  ArgmaxParams p{};
  p.tgt = target_logits;
  p.sb = sb;
  p.sg = sg;
  p.sp = sp;
  p.t_elems = R > 0 ? span({{B, sb}, {R, sg}}, V) : span({{B, sb}, {G, sg}, {k + 1, sp}}, V);
  p.tokens = tokens;
  p.B = B;
  p.G = G;
  p.k = k;
  p.V = V;
  p.R = rows_per_seq;
  p.row_of = row_of;
  p.parent = parent;
  p.path = path;
  p.best_g = best_g;
  p.accepted_len = accepted_len;
  p.out_tokens = out_tokens;
  p.ch = pl.ch;
  p.nch = pl.nch;
  p.div_seq = make_udiv(static_cast<unsigned int>(rows_per_seq) * static_cast<unsigned int>(pl.nch));
  p.div_nch = make_udiv(static_cast<unsigned int>(pl.nch));
  p.div_bg = make_udiv(static_cast<unsigned int>(B) * static_cast<unsigned int>(G));
  p.div_g = make_udiv(static_cast<unsigned int>(G));
  p.total = static_cast<unsigned int>(total);
  p.ctrl = ws.ctrl;
  p.seq = ws.seq;
  p.t_dtype = t_dtype;
  const ThreshLayout tl = threshold_layout(rows, pl.nch);
  if (thresh) {
    p.c2 = 1.4426950408889634f / temperature;
    p.log2_tau = std::log2(threshold);
    p.sslots = reinterpret_cast<unsigned long long*>(static_cast<unsigned char*>(ws.tail) + tl.sslots);
    p.rstats = reinterpret_cast<unsigned long long*>(static_cast<unsigned char*>(ws.tail) + tl.rstats);
  }
  const ArgLayout lay = argmax_layout(rows, pl.nch);
  unsigned char* tail = static_cast<unsigned char*>(ws.tail);
  p.slots = reinterpret_cast<unsigned long long*>(tail + lay.slots);
  p.rkey = reinterpret_cast<unsigned long long*>(tail + lay.rkey);
  p.rc = reinterpret_cast<unsigned int*>(tail + lay.rc);
  p.dead = reinterpret_cast<unsigned int*>(tail + lay.dead);
  cudaError_t e;
  if ((R == 0 || row_of) && !thresh && use_oneshot(rows * V * st)) {
    if (row_of) {
      // rows form: row r of sequence b sits at b sb + r sg.  The streaming
      // grid addresses row r as branch r / (k + 1), position r % (k + 1), so
      // a branch stride of (k + 1) sg and a position stride of sg reach it.
      p.sg = sg * (k + 1);
      p.sp = sg;
    }
    const int ch1 = oneshot_chunk_entries(t_dtype);
    p.nch1 = (V + ch1 - 1) / ch1;
    p.div_nch1 = make_udiv(static_cast<unsigned int>(p.nch1));
    p.div_R = make_udiv(static_cast<unsigned int>(rows_per_seq));
    if (rows * p.nch1 >= (1ll << 31)) return SV_ERR_INVALID_ARG;
    e = launch_argmax_oneshot(p, t_dtype, tma, static_cast<cudaStream_t>(stream));
  } else {
    e = launch_argmax(p, t_dtype, tma, grid, kernel_smem_bytes(),
                      static_cast<cudaStream_t>(stream));
  }
  return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

extern "C" int spec_verify_greedy(const void* target_logits, int t_dtype, int64_t t_stride_b,
                                  int64_t t_stride_pos, const int32_t* draft_tokens, int B, int k,
                                  int V, int32_t* accepted_len, int32_t* out_tokens,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return argmax_call(target_logits, t_dtype, t_stride_b, 0, t_stride_pos, draft_tokens, B, 1, k,
                     V, 0, nullptr, nullptr, nullptr, nullptr, accepted_len, out_tokens,
                     workspace, workspace_bytes, stream,
                     spec_verify_workspace_size(B, 1, k, V));
}

extern "C" int spec_verify_multi_candidate(const void* target_logits, int t_dtype,
                                           int64_t t_stride_b, int64_t t_stride_g,
                                           int64_t t_stride_pos, const int32_t* cand_tokens,
                                           int B, int G, int k, int V, int32_t* best_candidate,
                                           int32_t* accepted_len, int32_t* out_tokens,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream) {
  if (!best_candidate && B > 0) return SV_ERR_INVALID_ARG;
  return argmax_call(target_logits, t_dtype, t_stride_b, t_stride_g, t_stride_pos, cand_tokens, B,
                     G, k, V, 0, nullptr, nullptr, nullptr, best_candidate, accepted_len,
                     out_tokens, workspace, workspace_bytes, stream,
                     spec_verify_workspace_size(B, G, k, V));
}

extern "C" int spec_verify_multi_candidate_rows(const void* row_logits, int t_dtype,
                                                int64_t r_stride_b, int64_t r_stride_row,
                                                const int32_t* row_of,
                                                const int32_t* cand_tokens, int B, int G, int k,
                                                int R, int V, int32_t* best_candidate,
                                                int32_t* accepted_len, int32_t* out_tokens,
                                                void* workspace, size_t workspace_bytes,
                                                void* stream) {
  if (B > 0 && (!best_candidate || !row_of || R < 1)) return SV_ERR_INVALID_ARG;
  return argmax_call(row_logits, t_dtype, r_stride_b, r_stride_row, 0, cand_tokens, B, G, k, V,
                     B > 0 ? R : 0, B > 0 ? row_of : nullptr, nullptr, nullptr, best_candidate,
                     accepted_len, out_tokens, workspace, workspace_bytes, stream,
                     spec_verify_workspace_size(B, G, k, V));
}

extern "C" int spec_verify_threshold(const void* target_logits, int t_dtype, int64_t t_stride_b,
                                     int64_t t_stride_pos, const int32_t* draft_tokens, int B,
                                     int k, int V, float temperature, float threshold,
                                     int32_t* accepted_len, int32_t* out_tokens, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  if (!(temperature > 0.0f) || !std::isfinite(temperature) ||
      !std::isfinite(1.4426950408889634f / temperature))
    return SV_ERR_INVALID_ARG;
  if (!(threshold > 0.0f) || !(threshold <= 1.0f)) return SV_ERR_INVALID_ARG;
  return argmax_call(target_logits, t_dtype, t_stride_b, 0, t_stride_pos, draft_tokens, B, 1, k,
                     V, 0, nullptr, nullptr, nullptr, nullptr, accepted_len, out_tokens,
                     workspace, workspace_bytes, stream, spec_verify_workspace_size(B, 1, k, V),
                     temperature, threshold);
}

extern "C" size_t spec_verify_tree_workspace_size(int B, int N, int V) {
  if (B < 0 || N < 1 || N > 64 || V < 1) return 0;
  size_t tail = 0;
  for (int es : {2, 4}) {
    const long long rows = static_cast<long long>(B) * N;
    const size_t a = argmax_layout(rows, plan_chunks(rows, V, es, es, kArgmaxChunkBytes).nch).bytes;
    if (a > tail) tail = a;
  }
  const size_t total = kCtrlBytes + seq_bytes(B) + tail;
  return (total + 255) / 256 * 256;
}

extern "C" int spec_verify_tree_greedy(const void* node_logits, int t_dtype, int64_t stride_b,
                                       int64_t stride_node, const int32_t* parent,
                                       const int32_t* tokens, int B, int N, int V,
                                       int32_t* accepted_len, int32_t* path,
                                       int32_t* out_tokens, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (N < 1 || N > 64 || B < 0 || V < 1) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!parent || !tokens || !path) return SV_ERR_INVALID_ARG;
  // a tree of N nodes runs as one "sequence" of R = N rows of the argmax
  // machinery (G = 2, k = 31 only bound R by 64); the finalize walks the tree
  return argmax_call(node_logits, t_dtype, stride_b, stride_node, 0, tokens, B, 2, 31, V, N,
                     nullptr, parent, path, nullptr, accepted_len, out_tokens, workspace,
                     workspace_bytes, stream, spec_verify_tree_workspace_size(B, N, V));
}

extern "C" int spec_verify_commit(const int32_t* accepted_len, const int32_t* out_tokens, int B,
                                  int k, int32_t* seq_len, int32_t* token_buf,
                                  int64_t buf_stride, int capacity, int32_t* next_input,
                                  void* workspace, void* stream) {
  if (B < 0 || k < 0 || k > 32 || capacity < 0 || buf_stride < capacity) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!accepted_len || !out_tokens || !seq_len || (capacity > 0 && !token_buf))
    return SV_ERR_INVALID_ARG;
  if (!aligned(accepted_len, 4) || !aligned(out_tokens, 4) || !aligned(seq_len, 4) ||
      (token_buf && !aligned(token_buf, 4)) || (next_input && !aligned(next_input, 4)) ||
      (workspace && !aligned(workspace, 16)))
    return SV_ERR_MISALIGNED;
  const cudaError_t e = launch_commit(
      accepted_len, out_tokens, B, k, seq_len, token_buf, buf_stride, capacity, next_input,
      workspace ? reinterpret_cast<Ctrl*>(workspace) : nullptr, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}

extern "C" int spec_verify_philox4x32_10(const uint32_t* counters, int64_t n, uint64_t seed,
                                         uint32_t* out, void* stream) {
  if (n < 0 || (n > 0 && (!counters || !out))) return SV_ERR_INVALID_ARG;
  if (n == 0) return SV_OK;
  if (!aligned(counters, 16) || !aligned(out, 16)) return SV_ERR_MISALIGNED;
  const cudaError_t e = launch_philox(
      reinterpret_cast<const uint4*>(counters), n, static_cast<unsigned int>(seed & 0xffffffffull),
      static_cast<unsigned int>(seed >> 32), reinterpret_cast<uint4*>(out),
      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}
