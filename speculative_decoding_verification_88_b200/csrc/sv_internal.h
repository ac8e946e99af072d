// sv_internal.h -- parameter blocks and work plan shared by the C ABI layer
// (sv_api.cu) and the kernels (sv_kernels.cu).  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace sv {

// ---- CTA shape of the persistent verify kernels -------------------------
// warps 0..kProducerWarps-1: producers (one thread each: tickets, waits, bulk
//   copies), one per compute group in the stochastic kernel
// next kComputeWarps warps: compute (reduce one chunk held in shared memory)
// last kComputeGroups warps: epilogues, one per compute group (publish chunk
//   partials, merge rows, finalize sequences)
#ifndef SV_COMPUTE_WARPS
#define SV_COMPUTE_WARPS 16
#endif
constexpr int kComputeWarps = SV_COMPUTE_WARPS;
// The compute warps form two groups that take alternate ring stages, so one
// group's load and reduction latency overlaps the other group's arithmetic;
// each group has its own epilogue warp.
constexpr int kComputeGroups = 2;
constexpr int kGroupWarps = kComputeWarps / kComputeGroups;
// One producer warp per compute group (the argmax kernel uses the first).
constexpr int kProducerWarps = kComputeGroups;
constexpr int kThreads = 32 * (kProducerWarps + kComputeWarps + kComputeGroups);
constexpr int kComputeThreads = kGroupWarps * 32;  // threads that share one chunk
#ifndef SV_STAGES
#define SV_STAGES 4
#endif
#ifndef SV_STAGE_BYTES
#define SV_STAGE_BYTES (56 * 1024)
#endif
constexpr int kStages = SV_STAGES;          // ring stages per CTA, split evenly over the groups
constexpr int kStageBytes = SV_STAGE_BYTES;  // a multiple of 128
static_assert(kStageBytes % 128 == 0, "stages stay 128-byte aligned");

// Entries of a full chunk: as many as fit `bytes` at `bpe` bytes per entry,
// rounded down to whole rounds of 16-byte vectors over the kComputeThreads
// threads of a group for the narrowest tensor (es_min bytes per element), so
// that every thread holds the same number of vectors and no -inf padding is
// needed; a budget below one round falls back to a multiple of 8 entries.
__host__ __device__ constexpr int full_chunk_entries(int bytes, int bpe, int es_min) {
  return bytes / bpe >= kComputeThreads * 16 / es_min
             ? bytes / bpe / (kComputeThreads * 16 / es_min) * (kComputeThreads * 16 / es_min)
             : ((bytes / bpe) & ~7) > 8 ? (bytes / bpe) & ~7 : 8;
}

// Device-wide control words at the start of the workspace (256 bytes).
struct Ctrl {
  unsigned int ticket;    // next work ticket (phase 1 of stochastic verify)
  unsigned int exits;     // producers that took their last ticket
  unsigned int flags;     // sticky SV_FLAG_* bits
  unsigned int ticket2;   // stochastic: next phase-2 ticket
  unsigned int resolved;  // stochastic: sequences whose accepted length is known
  unsigned int pad[59];   // (all counters are reset by the last producer to leave)
};
static_assert(sizeof(Ctrl) == 256, "Ctrl must be 256 bytes");

// Per-sequence record (64 bytes), zero between calls: the kernel that sets
// a field also clears it.
struct SeqRec {
  unsigned int cnt1;         // argmax: rows merged
  unsigned int cnt2;         // stochastic: phase-2 chunks published
  unsigned long long state;  // stochastic: rows decided (bits 0..31), rows rejected (32..63)
  float mt, ist, md, isd;    // stochastic: row n max (log2 units) and 1/sum, of p and of q
  int n;                     // stochastic: accepted length
  unsigned int pad[7];
};
static_assert(sizeof(SeqRec) == 64, "SeqRec must be 64 bytes");

// Chunking of the vocabulary axis: `nch` chunks of `ch` elements (the last
// one shorter); ch is a multiple of 8 so that every chunk of a 16-byte
// aligned row starts 16-byte aligned for both 2- and 4-byte elements.
struct Plan {
  int ch;
  int nch;
};

// rows: rows (or row pairs) a call reduces; bpe: bytes per vocab entry of
// one unit of work (target + draft bytes for a stochastic pair); es_min: the
// narrowest element size in it; chunk_bytes: most bytes one chunk may take
// (at most a stage).  Chunks are full_chunk_entries long, the last one of a
// row shorter; small calls split rows finer.
Plan plan_chunks(long long rows, int V, int bpe, int es_min, int chunk_bytes);

// Chunk budgets.  Stochastic chunks fill a stage (56 KB measured faster than
// 48 KB: 230 -> 224 us on B = 256, k = 8, V = 128256); argmax chunks are
// smaller, since an argmax chunk is cheap to reduce and its calls are small
// enough that the ramp of the ring dominates (greedy B = 64, k = 4,
// V = 128256: 40 KB chunks 15.9 us, 48 KB 16.9 us, 54 KB 18.1 us).
constexpr int kStochChunkBytes = kStageBytes;
constexpr int kArgmaxChunkBytes = 40 * 1024 < kStageBytes ? 40 * 1024 : kStageBytes;

// Division of 31-bit values by a divisor fixed per call, as a multiply-high
// and a shift (Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994): with l = ceil(log2 d) and m = ceil(2^(31+l)/d),
// floor(n/d) = floor(n m / 2^(31+l)) for 0 <= n < 2^31, and m < 2^32.
struct UDiv {
  unsigned int d, m, shift;  // d == 1: m == 0, the quotient is n
};
inline UDiv make_udiv(unsigned int d) {
  UDiv u{d, 0u, 0u};
  if (d <= 1u) return u;
  unsigned int l = 0;
  while ((1ull << l) < d) ++l;
  u.m = static_cast<unsigned int>(((1ull << (31 + l)) + d - 1) / d);
  u.shift = l - 1;  // 31 + l - 32
  return u;
}

struct StochParams {
  const void* tgt;
  long long t_sb, t_sp;
  const void* drf;
  long long d_sb, d_sp;
  long long t_elems, d_elems;  // elements the target / draft views span (bounds checks)
  const int* tokens;  // [B, k]
  int B, k, V;
  float c2;    // log2(e) / T: logit -> log2-domain scale
  unsigned int key0, key1, seq_offset;
  int* accepted_len;
  int* out_tokens;
  float* probs;  // nullable
  int ch, nch;
  // Tickets.  Phase 1 (counter ticket): chunk t % nch of row pair t / nch,
  // position-major -- position i = row / B of sequence b = row % B -- so that
  // every sequence's pair i comes a whole position block (B nch tickets)
  // after its pair i - 1, late enough for a rejection before it to be known
  // and the pair to be retired unread.  Phase 2 (counter ticket2): chunk
  // t % nch of the sequence in ready-list entry t / nch, the list filled in
  // the order the sequences' accepted lengths become known.
  unsigned int total1;   // k B nch
  unsigned int total2;   // B nch
  int park;              // 1: producers park phase-1 chunks of undecided pairs
  UDiv div_nch, div_B;   // / nch, / B
  Ctrl* ctrl;
  SeqRec* seq;
  // Partials, published with one 64-bit store each and never zero once
  // written (so the value is its own "ready" flag):
  unsigned long long* p1;  // [B][k][nch][2]: chunk (max, sum) of target, of draft
  unsigned long long* r1;  // [B][k][2]: row (max, sum) of target, of draft; written for
                           // rejected rows only, for the sequence's resolution
  unsigned long long* p2;  // [B][nch]: chunk Gumbel-max key, 1 = no candidate
  unsigned int* rc;        // [B][k]: chunks of a row published
  unsigned long long* list;  // [B] ready list: (b + 1) | n << 32, in resolution order
};

struct ArgmaxParams {
  const void* tgt;
  long long sb, sg, sp;  // rows form: sg is the row stride, sp unused (one-grid path:
                         // sg = (k + 1) row strides, sp = one, so that row r = g (k + 1) + i
                         // sits at g sg + i sp)
  long long t_elems;     // elements the logits view spans (bounds checks)
  const int* tokens;     // [B, G, k]
  int B, G, k, V;
  int R;                 // rows per sequence: G * (k + 1), the distinct rows of the rows
                         // form, or the nodes of a tree
  const int* row_of;     // rows form: [B, G, k+1] row of (b, g, i); nullptr: row g*(k+1)+i
  const int* parent;     // tree form: [B, R] parent of each node (tokens and out_tokens
                         // are then [B, R]; G and k only bound R)
  int* path;             // tree form: [B, R] accepted path out
  // threshold acceptance (sslots != nullptr): row softmax statistics as well
  int t_dtype;                  // SV_F32 / SV_BF16 (the finalize reads draft-token logits)
  float c2;                     // log2(e) / T
  float log2_tau;               // lg2 of the acceptance threshold
  unsigned long long* sslots;   // [B][R][nch] chunk (max, sum) statistics
  unsigned long long* rstats;   // [B][R] row statistics
  int* best_g;  // nullable
  int* accepted_len;
  int* out_tokens;
  int ch, nch;
  // Ticket decode.  Plain mode (greedy, multi-candidate) is position-major:
  // ticket t is chunk t % nch of row t / nch, taken as (position, sequence,
  // branch) with the branch fastest, so that every branch's row i comes a
  // whole position block (B G nch tickets) after its row i - 1.  The other
  // modes go sequence by sequence: / (R * nch), then / nch.
  UDiv div_seq, div_nch, div_bg, div_g;  // / (R * nch), / nch, / (B * G), / G
  // One-shot form (small plain calls): nch1 chunks of a row per block grid.
  int nch1;
  UDiv div_nch1, div_R;  // / nch1, / R
  unsigned int total;
  Ctrl* ctrl;
  SeqRec* seq;
  unsigned long long* slots;  // [B][R][nch] chunk argmax keys
  unsigned long long* rkey;   // [B][R] row argmax keys
  unsigned int* rc;           // [B][R] chunks of a row published
  // Plain mode: per (sequence, branch), 64 - the smallest position found so
  // far whose draft differs from the row argmax (0: none yet).  Rows past it
  // decide nothing, and their chunks are retired without being read.
  unsigned int* dead;         // [B][G]
};

// dtype codes follow sv_dtype (0 = f32, 1 = bf16).  Return cudaError_t.
cudaError_t launch_stochastic(const StochParams& p, int t_dtype, int d_dtype, bool tma,
                              int grid, size_t smem, cudaStream_t stream);
cudaError_t launch_argmax(const ArgmaxParams& p, int t_dtype, bool tma, int grid, size_t smem,
                          cudaStream_t stream);
// Plain greedy / multi-candidate verify as one grid of row-chunk blocks (no
// persistent pipeline): every row is read and all of a block's loads are in
// flight at once; a second grid (a programmatic dependent launch) finalizes
// every sequence.
cudaError_t launch_argmax_oneshot(const ArgmaxParams& p, int t_dtype, bool vec, cudaStream_t st);
int oneshot_chunk_entries(int t_dtype);
cudaError_t launch_commit(const int* accepted_len, const int* out_tokens, int B, int k,
                          int* seq_len, int* token_buf, long long buf_stride, int capacity,
                          int* next_input, Ctrl* ctrl, cudaStream_t st);
cudaError_t launch_philox(const uint4* ctr, long long n, unsigned int key0, unsigned int key1,
                          uint4* out, cudaStream_t stream);
size_t kernel_smem_bytes();

// Kernels of this library launched in this process, counted when a launch
// returns success (a launch captured into a CUDA graph counts once, at
// capture).  Returns its argument, so a launcher can end with
// `return counted(cudaGetLastError(), n)`.
cudaError_t counted(cudaError_t e, int n);
unsigned long long launches_so_far();

}  // namespace sv
