// sv_tree_stoch.cu -- stochastic verify of a draft token tree (sm_100a).
//
// "Accelerating Sonar through speculation", section "EAGLE": the draft
// explores a tree of Top-K candidates per node, the longest acceptable path
// is kept and the target adds one token.  The siblings are fixed candidates,
// so the draft distribution behind each child is a point mass on its token;
// speculative rejection applied to the siblings in node order then accepts
// child c (token x) at node u with probability p_u(x) / R, R the target mass
// left after the siblings already rejected, and a node where every child was
// rejected draws the last token from p_u outside the rejected tokens E.  The
// committed tokens then follow the target at every depth.
//
// Three launches on the caller's stream:
//   tree_stats_kernel   one block per (node row, chunk): the chunk's softmax
//                       statistics (max and sum of 2^(l c2 - max), log2 units)
//                       from 16-byte vector loads, 8 in flight per thread;
//                       one exponential pair in four on the FMA pipe.
//   tree_walk_kernel    one warp per sequence: merges each node row's chunk
//                       statistics, gathers p(x) of every child under its
//                       parent's row and its acceptance draw (lane-parallel),
//                       then walks the tree with warp-uniform shuffles and
//                       ballots.  Writes the path and accepted tokens, and the
//                       final node and E for the draw.
//   tree_sample_kernel  one block per (sequence, 8192-entry piece) of the
//                       final node's row: Gumbel-max over l c2 outside E (and
//                       over the whole row as the fallback), merged by 64-bit
//                       atomicMax; the last block of a sequence writes the
//                       token.  The draw is issue-bound (a Philox block per
//                       four entries, two lg2 per entry) on one row per
//                       sequence; each thread loads all its vectors before
//                       it draws, so a block waits for DRAM once.
// Every workspace word written here is cleared again by the kernel that
// consumes it, so the workspace stays zero between calls of any mode.
#include <climits>
#include <cmath>
#include <cstdint>

#include "spec_verify.h"
#include "sv_device.cuh"

namespace sv {
namespace {

constexpr int kTsThreads = 256;
// 16-byte vectors per thread and chunk (4, i.e. 8192-entry bf16 chunks, was
// slower for the stochastic tree call: 120.5 against 109.9 us at B = 64,
// N = 26, V = 128256)
constexpr int kTsVecs = 8;
// One pair of exponentials in kTsPolyEvery runs on the FMA pipe
// (ex2_poly_x2), the rest on the special-function unit, which the statistics
// pass otherwise saturates.  1 in 8 / 4 / 3 / 2 / every pair (us per
// stochastic tree call at B = 64, N = 26, V = 128256): 106.9 / 101.7 /
// 104.3 / 110.5 / 128.4; all on the special-function unit 106.7.
constexpr int kTsPolyEvery = 4;
// Entries per block of the final draw, each thread's loads issued before its
// draws.  2048 / 4096 / 8192 / 12288 / 16384 entries: 111.9 / 108.2 / 106.9 /
// 108.1 / 108.7 us per stochastic tree call at B = 64, N = 26, V = 128256
// (1024 entries: 123.4).  Launching the walk and the draw as programmatic
// dependents of the grid before them was slower (116.9).
constexpr int kSampleEntries = 8192;
constexpr int kWalkWarps = 4;
constexpr int kMaxNodes = 64;

template <typename T>
__host__ __device__ constexpr int tree_chunk() {
  return kTsThreads * kTsVecs * Elem<T>::kPerVec;  // 16384 bf16 or 8192 f32 entries
}

// The final draw of one sequence (written by the walk, cleared by the draw).
struct TreeRec {
  int u, tag, n, ne;      // final node, Philox tag, accepted length, |E|
  int excl[kMaxNodes];    // E: the rejected tokens at u, in node order
};
static_assert(sizeof(TreeRec) % 16 == 0, "TreeRec keeps 16-byte alignment");

struct TreeStochParams {
  const void* logits;
  long long sb, sn;  // element strides of sequence and node
  long long l_elems;  // elements the logits view spans (bounds checks)
  const int* parent;
  const int* tokens;
  int B, N, V, nch;  // nch chunks per row (statistics)
  int nch_s;         // pieces of kSampleEntries per row (final draw)
  bool vec;          // every row starts 16-byte aligned
  float c2;          // log2(e) / T
  unsigned int key0, key1, seq_offset;
  int* accepted_len;
  int* path;
  int* out_tokens;
  Ctrl* ctrl;
  float2* part;              // [B*N][nch] chunk (max, sum)
  TreeRec* rec;              // [B]
  unsigned long long* keys;  // [B][2] best key outside E, best key of the row
  unsigned int* cnt;         // [B] chunks of the final row done
};

template <typename T>
__device__ __forceinline__ uint4 neg_inf_vec();
template <>
__device__ __forceinline__ uint4 neg_inf_vec<uint16_t>() {
  return make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
}
template <>
__device__ __forceinline__ uint4 neg_inf_vec<float>() {
  return make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u);
}

// --------------------------------------------------------- row statistics

template <typename T>
__global__ void __launch_bounds__(kTsThreads) tree_stats_kernel(TreeStochParams p) {
  dep_enter();
  constexpr int EPV = Elem<T>::kPerVec;
  constexpr int CH = tree_chunk<T>();
  const long long blk = blockIdx.x;
  const int c = static_cast<int>(blk % p.nch);
  const long long row = blk / p.nch;  // b * N + j
  const int b = static_cast<int>(row / p.N), j = static_cast<int>(row % p.N);
  const long long off = static_cast<long long>(b) * p.sb + static_cast<long long>(j) * p.sn;
  const int x0 = c * CH;
  int len = min(CH, p.V - x0);
  const int tid = threadIdx.x;
  if (!SV_IN(p.ctrl, row, static_cast<long long>(p.B) * p.N) ||
      !SV_IN_RANGE(p.ctrl, off + x0, len, p.l_elems))
    len = 0;  // (bounds-checked builds: a bad block reads nothing)
  float mx = -INFINITY, s = 0.0f;
  if (p.vec) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.logits) + off + x0);
    const int nv = len / EPV;
    uint4 v[kTsVecs];
#pragma unroll
    for (int q = 0; q < kTsVecs; ++q) {
      const int i = tid + q * kTsThreads;
      v[q] = i < nv ? __ldg(src + i) : neg_inf_vec<T>();
    }
    const int te = nv * EPV + tid;  // at most one ragged entry per thread
    const float tail = te < len ? load_elem<T>(p.logits, off + x0 + te) : -INFINITY;
#pragma unroll
    for (int q = 0; q < kTsVecs; ++q) mx = fmaxf(mx, vec_max<T>(v[q]));
    mx = fmaxf(mx, tail) * p.c2;
    if (mx != -INFINITY) {
      // pairs of entries: one f32x2 FMA for the exponents, one f32x2 add;
      // one pair in kTsPolyEvery on the FMA pipe
      const unsigned long long cc = pack2(p.c2, p.c2), mm = pack2(-mx, -mx);
      unsigned long long acc0 = 0ull, acc1 = 0ull;
#pragma unroll
      for (int q = 0; q < kTsVecs; ++q) {
        float f[EPV];
        unpack(v[q], f);
#pragma unroll
        for (int e = 0; e < EPV; e += 2) {
          float y0, y1;
          unpack2(fma2(pack2(f[e], f[e + 1]), cc, mm), y0, y1);
          const unsigned long long x = ((q * EPV + e) / 2) % kTsPolyEvery == kTsPolyEvery - 1
                                           ? ex2_poly_x2(y0, y1)
                                           : pack2(ex2f(y0), ex2f(y1));
          if ((e & 2) == 0) acc0 = add2(acc0, x);
          else acc1 = add2(acc1, x);
        }
      }
      float a0, a1, b0, b1;
      unpack2(acc0, a0, a1);
      unpack2(acc1, b0, b1);
      s = ((a0 + a1) + (b0 + b1)) + ex2f(fmaf(tail, p.c2, -mx));
    }
  } else {
    for (int e = tid; e < len; e += kTsThreads) mx = fmaxf(mx, load_elem<T>(p.logits, off + x0 + e));
    mx *= p.c2;
    if (mx != -INFINITY)
      for (int e = tid; e < len; e += kTsThreads)
        s += ex2f(fmaf(load_elem<T>(p.logits, off + x0 + e), p.c2, -mx));
  }
  // block merge: warps first (max, then rescaled sums), then the 8 warps
  __shared__ float s_m[kTsThreads / 32], s_s[kTsThreads / 32];
  const float wm = warp_max(mx);
  const float ws = warp_sum(mx == -INFINITY ? 0.0f : s * ex2f(mx - wm));
  if ((tid & 31) == 0) {
    s_m[tid >> 5] = wm;
    s_s[tid >> 5] = ws;
  }
  __syncthreads();
  if (tid == 0) {
    float M = -INFINITY, S = 0.0f;
#pragma unroll
    for (int w = 0; w < kTsThreads / 32; ++w) merge_stats(M, S, s_m[w], s_s[w]);
    p.part[row * p.nch + c] = make_float2(M, S);
  }
}

// --------------------------------------------------------------- tree walk

// Value v of node c, held by lane c % 32 in slot c / 32 (c warp-uniform).
template <typename V>
__device__ __forceinline__ V node_value(const V (&v)[2], int c) {
  const V a = __shfl_sync(0xffffffffu, v[0], c & 31);
  const V b = __shfl_sync(0xffffffffu, v[1], c & 31);
  return c < 32 ? a : b;
}

template <typename T>
__global__ void __launch_bounds__(32 * kWalkWarps) tree_walk_kernel(TreeStochParams p) {
  dep_enter();
  __shared__ float s_m[kWalkWarps][kMaxNodes], s_is[kWalkWarps][kMaxNodes];
  __shared__ int s_path[kWalkWarps][kMaxNodes];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * kWalkWarps + w;
  if (b >= p.B) return;  // whole warps only; no block barrier below
  const int N = p.N;
  const long long nb = static_cast<long long>(b) * N;

  // 1. statistics of every node row (the chunk partials are cleared)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = lane + 32 * h;
    if (j < N) {
      float M = -INFINITY, S = 0.0f;
      float2* pp = p.part + (nb + j) * p.nch;
      for (int c = 0; c < p.nch; ++c) {
        const float2 v = pp[c];
        merge_stats(M, S, v.x, v.y);
        pp[c] = make_float2(0.0f, 0.0f);
      }
      s_m[w][j] = M;
      s_is[w][j] = 1.0f / S;
    }
  }
  __syncwarp();

  // 2. per node j >= 1: parent, token, p_parent(token) and acceptance draw
  const unsigned int seq = static_cast<unsigned int>(b) + p.seq_offset;
  int par[2], xs[2];
  float pr[2], ua[2];
  bool bad_parent = false;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = lane + 32 * h;
    par[h] = -1;
    xs[h] = -1;
    pr[h] = 0.0f;
    ua[h] = 1.0f;
    if (j >= 1 && j < N) {
      const int q = p.parent[nb + j];
      const int x = p.tokens[nb + j];
      xs[h] = x;
      if (q < 0 || q >= j) {
        bad_parent = true;
      } else {
        par[h] = q;
        if (x >= 0 && x < p.V &&
            SV_IN(p.ctrl, static_cast<long long>(b) * p.sb + static_cast<long long>(q) * p.sn + x,
                  p.l_elems)) {
          const float l = load_elem<T>(p.logits, static_cast<long long>(b) * p.sb +
                                                     static_cast<long long>(q) * p.sn + x);
          pr[h] = ex2f(fmaf(l, p.c2, -s_m[w][q])) * s_is[w][q];
        }
      }
      ua[h] = accept_uniform(
          philox10(make_uint4(0u, static_cast<uint32_t>(j - 1), seq, kTagAccept), p.key0, p.key1).x);
    }
  }
  if (__any_sync(0xffffffffu, bad_parent) && lane == 0) atomicOr(&p.ctrl->flags, kFlagInvalidTree);

  // 3. the walk; every value below is warp-uniform
  int u = 0, n = 0;
  unsigned long long E = 0ull;  // rejected children of u whose tokens form E
  bool has_child = false, bad_token = false;
  if (lane == 0) s_path[w][0] = 0;
  for (;;) {
    unsigned long long kids = static_cast<unsigned long long>(__ballot_sync(0xffffffffu, par[0] == u)) |
                              (static_cast<unsigned long long>(__ballot_sync(0xffffffffu, par[1] == u)) << 32);
    has_child = kids != 0ull;
    E = 0ull;
    float R = 1.0f;
    int next = -1;
    while (kids) {
      const int c = __ffsll(static_cast<long long>(kids)) - 1;
      kids &= kids - 1ull;
      const int xc = node_value(xs, c);
      const float pc = node_value(pr, c);
      const float uc = node_value(ua, c);
      const bool valid = xc >= 0 && xc < p.V;
      bad_token |= !valid;
      const bool rep = (((E >> lane) & 1ull) && xs[0] == xc) ||
                       (((E >> (lane + 32)) & 1ull) && xs[1] == xc);
      const bool open = valid && !__any_sync(0xffffffffu, rep);
      if (open && uc * R < pc) {
        next = c;
        break;
      }
      if (open) {
        E |= 1ull << c;
        R -= pc;
      }
    }
    if (next < 0) break;
    u = next;
    ++n;
    if (lane == 0) s_path[w][n] = u;
  }
  __syncwarp();
  if (bad_token && lane == 0) atomicOr(&p.ctrl->flags, kFlagInvalidToken);

  // 4. outputs; out_tokens[b][n] comes from the draw
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = lane + 32 * h;
    if (j < N) {
      p.path[nb + j] = j <= n ? s_path[w][j] : -1;
      if (j != n) p.out_tokens[nb + j] = j < n ? p.tokens[nb + s_path[w][j + 1]] : -1;
      if ((E >> j) & 1ull) p.rec[b].excl[__popcll(E & ((1ull << j) - 1ull))] = xs[h];
    }
  }
  if (lane == 0) {
    p.accepted_len[b] = n;
    TreeRec& r = p.rec[b];
    r.u = u;
    r.tag = has_child ? static_cast<int>(kTagCorrection) : static_cast<int>(kTagBonus);
    r.n = n;
    r.ne = __popcll(E);
  }
}

// ------------------------------------------------------------ final draw

template <typename T>
__global__ void __launch_bounds__(kTsThreads) tree_sample_kernel(TreeStochParams p) {
  dep_enter();
  constexpr int EPV = Elem<T>::kPerVec;
  constexpr int CH = kSampleEntries;
  // E (the rejected tokens at the final node) as a bitmap over this block's
  // entries: one shared-memory word per 32 entries
  __shared__ uint32_t s_emask[CH / 32];
  __shared__ unsigned long long s_ke[kTsThreads / 32], s_ka[kTsThreads / 32];
  const int c = static_cast<int>(blockIdx.x % p.nch_s);
  const int b = static_cast<int>(blockIdx.x / p.nch_s);
  const int tid = threadIdx.x;
  TreeRec& rec = p.rec[b];
  const int u = rec.u, ne = min(rec.ne, kMaxNodes);
  const uint32_t tag = static_cast<uint32_t>(rec.tag);
  const int x0 = c * CH;
  for (int w = tid; w < CH / 32; w += kTsThreads) s_emask[w] = 0u;
  __syncthreads();
  if (tid < ne) {
    const int xe = rec.excl[tid] - x0;
    if (xe >= 0 && xe < CH) atomicOr(&s_emask[xe >> 5], 1u << (xe & 31));
  }
  __syncthreads();

  const long long off = static_cast<long long>(b) * p.sb + static_cast<long long>(u) * p.sn;
  const uint32_t seq = static_cast<uint32_t>(b) + p.seq_offset;
  int len = min(CH, p.V - x0);
  if (!SV_IN(p.ctrl, u, p.N) ||
      !SV_IN_RANGE(p.ctrl, off + x0, len, p.l_elems))
    len = 0;  // (bounds-checked builds: a bad block reads nothing)
  float bv = -INFINITY, av = -INFINITY;  // best outside E, best of the row
  int bi = INT_MAX, ai = INT_MAX;
  // entries arrive in increasing x: a strict > keeps the first maximum
  auto take = [&](float sc, bool in_e, int x) {
    const bool wa = sc > av, wb = sc > bv && !in_e;
    av = wa ? sc : av;
    ai = wa ? x : ai;
    bv = wb ? sc : bv;
    bi = wb ? x : bi;
  };
  auto words = [&](int x) {
    return philox10(make_uint4(static_cast<uint32_t>(x) >> 2, static_cast<uint32_t>(u), seq, tag),
                    p.key0, p.key1);
  };
  auto score1 = [&](float l, uint32_t word) {
    return fmaf(l, p.c2, gumbel_log2(neg_exp1_log2(word)));
  };
  if (p.vec) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.logits) + off + x0);
    const int nv = len / EPV;
    // every load of the thread first, then the draws
    constexpr int NV = (CH / EPV + kTsThreads - 1) / kTsThreads;
    uint4 raw[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = tid + j * kTsThreads;
      raw[j] = i < nv ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = tid + j * kTsThreads;
      if (i >= nv) break;
      float f[EPV];
      unpack(raw[j], f);
      const int e0 = i * EPV;
      const uint32_t m = s_emask[e0 >> 5] >> (e0 & 31);  // EPV bits, one word (EPV | 32)
#pragma unroll
      for (int g = 0; g < EPV / 4; ++g) {
        const uint4 wd = words(x0 + e0 + 4 * g);
        float ev[4], sc[4];
        neg_exp1_log2_x2(wd.x, wd.y, ev[0], ev[1]);
        neg_exp1_log2_x2(wd.z, wd.w, ev[2], ev[3]);
#pragma unroll
        for (int q = 0; q < 4; ++q) sc[q] = fmaf(f[4 * g + q], p.c2, gumbel_log2(ev[q]));
#pragma unroll
        for (int q = 0; q < 4; ++q) take(sc[q], (m >> (4 * g + q)) & 1u, x0 + e0 + 4 * g + q);
      }
    }
    const int te = nv * EPV + tid;
    if (te < len) {
      const int x = x0 + te;
      take(score1(load_elem<T>(p.logits, off + x), word_of(words(x), x & 3)),
           (s_emask[te >> 5] >> (te & 31)) & 1u, x);
    }
  } else {
    for (int e = tid; e < len; e += kTsThreads) {
      const int x = x0 + e;
      take(score1(load_elem<T>(p.logits, off + x), word_of(words(x), x & 3)),
           (s_emask[e >> 5] >> (e & 31)) & 1u, x);
    }
  }
  warp_argmax(bv, bi);
  warp_argmax(av, ai);
  if ((tid & 31) == 0) {
    s_ke[tid >> 5] = bv == -INFINITY ? 0ull : make_key(bv, bi);
    s_ka[tid >> 5] = av == -INFINITY ? 0ull : make_key(av, ai);
  }
  __syncthreads();
  if (tid == 0) {
    unsigned long long ke = 0ull, ka = 0ull;
#pragma unroll
    for (int w = 0; w < kTsThreads / 32; ++w) {
      ke = s_ke[w] > ke ? s_ke[w] : ke;
      ka = s_ka[w] > ka ? s_ka[w] : ka;
    }
    if (ke) atomicMax(&p.keys[2 * b], ke);
    if (ka) atomicMax(&p.keys[2 * b + 1], ka);
    __threadfence();
    if (atomicAdd(&p.cnt[b], 1u) == static_cast<unsigned int>(p.nch_s) - 1u) {
      __threadfence();
      ke = atomicExch(&p.keys[2 * b], 0ull);
      ka = atomicExch(&p.keys[2 * b + 1], 0ull);
      p.cnt[b] = 0u;
      int y;
      if (ke) {
        y = key_index(ke);
      } else {  // nothing outside E (rounding only): draw from the whole row
        y = ka ? key_index(ka) : -1;
        atomicOr(&p.ctrl->flags, kFlagResidualFallback);
      }
      p.out_tokens[static_cast<long long>(b) * p.N + rec.n] = y;
      for (int e = 0; e < ne; ++e) rec.excl[e] = 0;
      rec.u = 0;
      rec.tag = 0;
      rec.n = 0;
      rec.ne = 0;
    }
  }
}

// ------------------------------------------------------------------- host

struct TreeLayout {
  size_t part, rec, keys, cnt, total;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Chunks per row: the f32 chunk is the smaller, so its count bounds both.
int tree_nch(int V, int es) {
  const int ch = es == 2 ? tree_chunk<uint16_t>() : tree_chunk<float>();
  return (V + ch - 1) / ch;
}

TreeLayout tree_layout(int B, int N, int V) {
  TreeLayout l{};
  const size_t nch = static_cast<size_t>(tree_nch(V, 4));
  l.part = align_up(sizeof(Ctrl), 256);
  l.rec = align_up(l.part + static_cast<size_t>(B) * N * nch * sizeof(float2), 256);
  l.keys = align_up(l.rec + static_cast<size_t>(B) * sizeof(TreeRec), 256);
  l.cnt = align_up(l.keys + static_cast<size_t>(B) * 2 * sizeof(unsigned long long), 256);
  l.total = align_up(l.cnt + static_cast<size_t>(B) * sizeof(unsigned int), 256);
  return l;
}

bool is_aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

template <typename T>
cudaError_t launch_tree_stoch(const TreeStochParams& p, cudaStream_t st) {
  const long long rows = static_cast<long long>(p.B) * p.N;
  cudaError_t e = counted(launch_k(SV_PDL >= 2, tree_stats_kernel<T>,
                                   dim3(static_cast<unsigned int>(rows * p.nch)),
                                   dim3(kTsThreads), 0, st, p),
                          1);
  if (e != cudaSuccess) return e;
  e = counted(launch_k(SV_PDL >= 2, tree_walk_kernel<T>, dim3((p.B + kWalkWarps - 1) / kWalkWarps),
                       dim3(32 * kWalkWarps), 0, st, p),
              1);
  if (e != cudaSuccess) return e;
  return counted(launch_k(SV_PDL >= 2, tree_sample_kernel<T>,
                          dim3(static_cast<unsigned int>(static_cast<long long>(p.B) * p.nch_s)),
                          dim3(kTsThreads), 0, st, p),
                 1);
}

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" size_t spec_verify_tree_stochastic_workspace_size(int B, int N, int V) {
  if (B < 0 || N < 1 || N > kMaxNodes || V < 1) return 0;
  return tree_layout(B, N, V).total;
}

extern "C" int spec_verify_tree_stochastic(const void* node_logits, int t_dtype, int64_t stride_b,
                                           int64_t stride_node, const int32_t* parent,
                                           const int32_t* tokens, int B, int N, int V,
                                           float temperature, uint64_t seed,
                                           uint32_t seq_offset, int32_t* accepted_len,
                                           int32_t* path, int32_t* out_tokens, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  if (B < 0 || N < 1 || N > kMaxNodes || V < 1) return SV_ERR_INVALID_ARG;
  if (t_dtype != SV_F32 && t_dtype != SV_BF16) return SV_ERR_INVALID_ARG;
  if (!(temperature > 0.0f) || !std::isfinite(temperature) || !std::isnormal(temperature))
    return SV_ERR_INVALID_ARG;
  if (stride_b < 0 || stride_node < 0) return SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!node_logits || !parent || !tokens || !accepted_len || !path || !out_tokens || !workspace)
    return SV_ERR_INVALID_ARG;
  const int es = t_dtype == SV_BF16 ? 2 : 4;
  if (!is_aligned(node_logits, es) || !is_aligned(parent, 4) || !is_aligned(tokens, 4) ||
      !is_aligned(accepted_len, 4) || !is_aligned(path, 4) || !is_aligned(out_tokens, 4) ||
      !is_aligned(workspace, 16))
    return SV_ERR_MISALIGNED;
  const TreeLayout lay = tree_layout(B, N, V);
  if (workspace_bytes < lay.total) return SV_ERR_WORKSPACE;
  const int nch = tree_nch(V, es);
  const int nch_s = (V + kSampleEntries - 1) / kSampleEntries;
  if (static_cast<long long>(B) * N * nch >= (1ll << 31) ||
      static_cast<long long>(B) * nch_s >= (1ll << 31))
    return SV_ERR_INVALID_ARG;

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  TreeStochParams p{};
  p.logits = node_logits;
  p.sb = stride_b;
  p.sn = stride_node;
  p.l_elems = (static_cast<long long>(B) - 1) * stride_b + (static_cast<long long>(N) - 1) * stride_node + V;
  p.parent = parent;
  p.tokens = tokens;
  p.B = B;
  p.N = N;
  p.V = V;
  p.nch = nch;
  p.nch_s = nch_s;
  p.vec = is_aligned(node_logits, 16) && (stride_b * es) % 16 == 0 && (stride_node * es) % 16 == 0;
  p.c2 = 1.4426950408889634f / temperature;
  p.key0 = static_cast<unsigned int>(seed & 0xffffffffull);
  p.key1 = static_cast<unsigned int>(seed >> 32);
  p.seq_offset = seq_offset;
  p.accepted_len = accepted_len;
  p.path = path;
  p.out_tokens = out_tokens;
  p.ctrl = reinterpret_cast<Ctrl*>(ws);
  p.part = reinterpret_cast<float2*>(ws + lay.part);
  p.rec = reinterpret_cast<TreeRec*>(ws + lay.rec);
  p.keys = reinterpret_cast<unsigned long long*>(ws + lay.keys);
  p.cnt = reinterpret_cast<unsigned int*>(ws + lay.cnt);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = t_dtype == SV_BF16 ? launch_tree_stoch<uint16_t>(p, st)
                                           : launch_tree_stoch<float>(p, st);
  return e == cudaSuccess ? SV_OK : SV_ERR_CUDA;
}
