// sv_kernels.cu -- persistent verify kernels for sm_100a.
//
// One CTA per SM runs until the work tickets run out.  A ticket names one
// chunk of one row (or row pair); the vocabulary of every row is split into
// `nch` chunks so that a (sequence, position) row is reduced by many CTAs.
//
//   warp 0, lane 0   producer: takes tickets (atomicAdd), waits where a chunk
//                    depends on an earlier result, and streams the chunk into
//                    a 4-stage shared-memory ring with 1-D bulk copies (TMA,
//                    cp.async.bulk) that complete on an mbarrier.
//   warps 1..8       compute: reduce the chunk held in shared memory (softmax
//                    statistics, Gumbel-max, or argmax) to one record per warp.
//   last warp        epilogue: merges the warp records, publishes the chunk's
//                    partial to the workspace, counts arrivals per sequence,
//                    and, in the CTA that completes a sequence, finalizes it.
//
// Stochastic verify ("Accelerating Sonar through speculation", section
// "Draft-Target": acceptance compares the full draft and target
// distributions; the target's logits after the accepted prefix are sampled)
// runs in two phases keyed on the same ticket counter:
//   phase 1  chunks of row pairs (target i, draft i), i < k: per-chunk
//            online softmax statistics (max, sum of 2^(x*log2e/T - max)).
//            The last chunk of a sequence merges them, gathers p_i(x_i) and
//            q_i(x_i), draws u_i (Philox, tag ACCEPT), finds the first
//            rejection n with a warp ballot and publishes n.
//   phase 2  the `nch` chunks of the row that gives the next token: the row
//            pair n (correction, Gumbel-max over ln max(0, p_n - q_n)) or
//            target row k (bonus, Gumbel-max over l_k / T).  They are placed
//            `lag` sequences after their phase-1 chunks, so the pair is
//            usually still in L2 and the producer rarely waits.
// Target row k is read only for sequences that accept all k drafts.
//
// Greedy and multi-candidate verify ("Lookahead decoding" news piece,
// section "Lookahead decoding breaks the order dependency") are one phase:
// per-chunk argmax keys merged with a 64-bit atomicMax per row; the last
// chunk of a sequence compares every branch's drafts with its row argmaxes
// (warp ballot) and commits the longest branch.
//
// Every wait is bounded (kWaitLimitNs); on expiry the kernel raises
// kFlagTimeout, every role leaves its loop, and the producer waits for its
// bulk copies in flight before the CTA exits.  A CTA only ever waits for
// tickets smaller than the one it holds, and those are held by running CTAs,
// so the waits end.
#include <climits>

#include "sv_device.cuh"

namespace sv {

enum : int { kKindEnd = 0, kKindStats = 1, kKindCorrection = 2, kKindBonus = 3, kKindArgmax = 4 };

constexpr int kComputeThreads = kComputeWarps * 32;

struct Hdr {
  int kind;
  int b;       // sequence
  int i;       // position (stochastic) or row within the sequence (argmax)
  int c;       // chunk
  int x0;      // first vocabulary entry of the chunk
  int len;     // entries in the chunk
  int nvec_t;  // full 16-byte target vectors in shared memory
  int nvec_d;  // full 16-byte draft vectors in shared memory
  float mt, ist, md, isd;  // correction: row-n statistics
  long long toff;          // element offset of entry x0 in the target
  long long doff;          // element offset of entry x0 in the draft
};

struct Shared {
  uint64_t full[kStages];   // producer -> compute (bulk-copy bytes)
  uint64_t empty[kStages];  // epilogue -> producer (slot free)
  uint64_t rfull[kStages];  // compute -> epilogue (warp records written)
  Hdr hdr[kStages];
  float4 res[kStages][kComputeWarps];
};

constexpr size_t kSharedHead = (sizeof(Shared) + 127) / 128 * 128;

size_t kernel_smem_bytes() { return kSharedHead + static_cast<size_t>(kStages) * kStageBytes; }

// ------------------------------------------------------------------ waits

__device__ __forceinline__ bool wait_flag(const unsigned int* flag, Ctrl* ctrl) {
  if (ld_acquire_u32(flag)) return true;
  const unsigned long long t0 = global_ns();
  for (unsigned int spin = 1;; ++spin) {
    __nanosleep(32);
    if (ld_acquire_u32(flag)) return true;
    if ((spin & 63u) == 0u) {
      if (aborted(ctrl)) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicOr(&ctrl->flags, kFlagTimeout);
        return false;
      }
    }
  }
}

// After an abort: wait (bounded, ignoring the abort flag) until the last
// bulk copy issued into every stage has landed, so none writes shared memory
// after the CTA exits.
__device__ void drain_stages(Shared& sh, uint32_t uses) {
  for (uint32_t s = 0; s < static_cast<uint32_t>(kStages) && s < uses; ++s) {
    const uint32_t last = s + ((uses - 1 - s) / kStages) * kStages;
    const uint32_t parity = (last / kStages) & 1u;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(&sh.full[s], parity)) {
      if (global_ns() - t0 > 100000000ull) break;
    }
  }
}

__device__ __forceinline__ void leave_grid(Ctrl* ctrl) {
  // The last CTA to take its final ticket rewinds the ticket counter.
  if (atomicAdd(&ctrl->exits, 1u) == gridDim.x - 1) {
    atomicExch(&ctrl->ticket, 0u);
    atomicExch(&ctrl->exits, 0u);
  }
}

// Fill stage `s` with the chunk described by `h` (bulk copies of the full
// 16-byte vectors; the ragged end is read by the compute warps directly).
template <typename TT, typename TD, bool kTma>
__device__ __forceinline__ void issue_chunk(Shared& sh, unsigned char* stage, int s, Hdr& h,
                                            const void* tgt, const void* drf, int ch,
                                            bool with_draft) {
  h.nvec_t = kTma ? (h.len * Elem<TT>::kBytes) / 16 : 0;
  h.nvec_d = (kTma && with_draft) ? (h.len * Elem<TD>::kBytes) / 16 : 0;
  sh.hdr[s] = h;
  if (kTma) {
    const uint32_t bt = static_cast<uint32_t>(h.nvec_t) * 16u;
    const uint32_t bd = static_cast<uint32_t>(h.nvec_d) * 16u;
    mbar_arrive_expect_tx(&sh.full[s], bt + bd);
    if (bt) bulk_load(stage, reinterpret_cast<const TT*>(tgt) + h.toff, bt, &sh.full[s]);
    if (bd)
      bulk_load(stage + static_cast<size_t>(ch) * Elem<TT>::kBytes,
                reinterpret_cast<const TD*>(drf) + h.doff, bd, &sh.full[s]);
  } else {
    mbar_arrive(&sh.full[s]);
  }
}

// ------------------------------------------------------- chunk reductions

// Softmax statistics of one chunk, per warp: m = max(x) * c2 (log2 units)
// and s = sum 2^(x * c2 - m).  Vectors [0, nvec) come from shared memory,
// the remaining entries [nvec * EPV, len) from global memory.
template <typename T>
__device__ __forceinline__ void chunk_stats(const unsigned char* smem, int nvec, const void* g,
                                            long long goff, int len, float c2, int tid,
                                            float& m_out, float& s_out) {
  constexpr int EPV = Elem<T>::kPerVec;
  const uint4* sv = reinterpret_cast<const uint4*>(smem);
  float m = -INFINITY;
#pragma unroll 4
  for (int v = tid; v < nvec; v += kComputeThreads) m = fmaxf(m, vec_max<T>(sv[v]));
  for (int e = nvec * EPV + tid; e < len; e += kComputeThreads)
    m = fmaxf(m, load_elem<T>(g, goff + e));
  m = warp_max(m);
  float s = 0.0f, mc = -INFINITY;
  if (m != -INFINITY) {
    mc = m * c2;
#pragma unroll 4
    for (int v = tid; v < nvec; v += kComputeThreads) {
      float f[EPV];
      unpack(sv[v], f);
#pragma unroll
      for (int j = 0; j < EPV; ++j) s += ex2f(fmaf(f[j], c2, -mc));
    }
    for (int e = nvec * EPV + tid; e < len; e += kComputeThreads)
      s += ex2f(fmaf(load_elem<T>(g, goff + e), c2, -mc));
    s = warp_sum(s);
  }
  m_out = mc;
  s_out = s;
}

// Eight consecutive entries (group j of the chunk) from shared memory.
template <typename T>
__device__ __forceinline__ void load8(const unsigned char* smem, int j, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<uint16_t>(const unsigned char* smem, int j, float (&f)[8]) {
  unpack(reinterpret_cast<const uint4*>(smem)[j], f);
}
template <>
__device__ __forceinline__ void load8<float>(const unsigned char* smem, int j, float (&f)[8]) {
  const uint4* sv = reinterpret_cast<const uint4*>(smem);
  const uint4 a = sv[2 * j], b = sv[2 * j + 1];
  f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
  f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
  f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
  f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
}

struct Draw {
  uint32_t key0, key1, pos, seq, tag;
};

__device__ __forceinline__ uint4 vocab_words(const Draw& d, uint32_t c0) {
  return philox10(make_uint4(c0, d.pos, d.seq, d.tag), d.key0, d.key1);
}

// p(x) - q(x) from the logits and the row statistics.  Both products are
// rounded on their own (no fused multiply-add), so identical target and
// draft rows give exactly zero.
__device__ __forceinline__ float residual(float lt, float ld, float c2, const Hdr& h) {
  return __fmul_rn(ex2f(fmaf(lt, c2, -h.mt)), h.ist) - __fmul_rn(ex2f(fmaf(ld, c2, -h.md)), h.isd);
}

// Gumbel-max over the positive residual r(x) = p(x) - q(x) of one chunk:
// score ln r(x) + g(x).  Returns the warp's best (score, x); x = INT_MAX if
// the warp saw no positive residual.
template <typename TT, typename TD, bool kTma>
__device__ __forceinline__ void chunk_residual(const unsigned char* ts, const unsigned char* ds,
                                               const Hdr& h, const void* tgt, const void* drf,
                                               float c2, const Draw& d, int tid, float& bv,
                                               int& bi) {
  bv = -INFINITY;
  bi = INT_MAX;
  const int ng = kTma ? h.len / 8 : 0;
  for (int j = tid; j < ng; j += kComputeThreads) {
    float lt[8], ld[8], r[8];
    load8<TT>(ts, j, lt);
    load8<TD>(ds, j, ld);
    bool any = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      r[e] = residual(lt[e], ld[e], c2, h);
      any |= r[e] > 0.0f;
    }
    if (any) {
      const int xg = h.x0 + 8 * j;
      const uint4 w0 = vocab_words(d, static_cast<uint32_t>(xg) >> 2);
      const uint4 w1 = vocab_words(d, (static_cast<uint32_t>(xg) >> 2) + 1u);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (r[e] > 0.0f) {
          const float sc = lg2f(r[e]) * kLn2 + gumbel(word_of(e < 4 ? w0 : w1, e & 3));
          if (better(sc, xg + e, bv, bi)) {
            bv = sc;
            bi = xg + e;
          }
        }
      }
    }
  }
  for (int e = 8 * ng + tid; e < h.len; e += kComputeThreads) {
    const int x = h.x0 + e;
    const float r = residual(load_elem<TT>(tgt, h.toff + e), load_elem<TD>(drf, h.doff + e), c2, h);
    if (r > 0.0f) {
      const float sc = lg2f(r) * kLn2 +
                       gumbel(word_of(vocab_words(d, static_cast<uint32_t>(x) >> 2), x & 3));
      if (better(sc, x, bv, bi)) {
        bv = sc;
        bi = x;
      }
    }
  }
  warp_argmax(bv, bi);
}

// Gumbel-max over l(x) / T of one chunk of the bonus row.
template <typename TT, bool kTma>
__device__ __forceinline__ void chunk_bonus(const unsigned char* ts, const Hdr& h,
                                            const void* tgt, float invT, const Draw& d, int tid,
                                            float& bv, int& bi) {
  bv = -INFINITY;
  bi = INT_MAX;
  const int ng = kTma ? h.len / 8 : 0;
  for (int j = tid; j < ng; j += kComputeThreads) {
    float lt[8];
    load8<TT>(ts, j, lt);
    const int xg = h.x0 + 8 * j;
    const uint4 w0 = vocab_words(d, static_cast<uint32_t>(xg) >> 2);
    const uint4 w1 = vocab_words(d, (static_cast<uint32_t>(xg) >> 2) + 1u);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float sc = fmaf(lt[e], invT, gumbel(word_of(e < 4 ? w0 : w1, e & 3)));
      if (better(sc, xg + e, bv, bi)) {
        bv = sc;
        bi = xg + e;
      }
    }
  }
  for (int e = 8 * ng + tid; e < h.len; e += kComputeThreads) {
    const int x = h.x0 + e;
    const float sc = fmaf(load_elem<TT>(tgt, h.toff + e), invT,
                          gumbel(word_of(vocab_words(d, static_cast<uint32_t>(x) >> 2), x & 3)));
    if (better(sc, x, bv, bi)) {
      bv = sc;
      bi = x;
    }
  }
  warp_argmax(bv, bi);
}

// Argmax (first maximum) of one chunk.
template <typename T>
__device__ __forceinline__ void chunk_argmax(const unsigned char* smem, const Hdr& h,
                                             const void* g, int tid, float& bv, int& bi) {
  constexpr int EPV = Elem<T>::kPerVec;
  const uint4* sv = reinterpret_cast<const uint4*>(smem);
  float best = -INFINITY;
  int bvec = -1;
#pragma unroll 4
  for (int v = tid; v < h.nvec_t; v += kComputeThreads) {
    const float m = vec_max<T>(sv[v]);
    if (bvec < 0 || m > best) {
      best = m;
      bvec = v;
    }
  }
  int idx = INT_MAX;
  if (bvec >= 0) {
    float f[EPV];
    unpack(sv[bvec], f);
#pragma unroll
    for (int j = EPV - 1; j >= 0; --j)
      if (f[j] == best) idx = h.x0 + bvec * EPV + j;
  }
  for (int e = h.nvec_t * EPV + tid; e < h.len; e += kComputeThreads) {
    const float v = load_elem<T>(g, h.toff + e);
    if (better(v, h.x0 + e, best, idx)) {
      best = v;
      idx = h.x0 + e;
    }
  }
  warp_argmax(best, idx);
  bv = best;
  bi = idx;
}

// ============================================================ stochastic

template <typename TT, typename TD, bool kTma>
__device__ void stoch_producer(const StochParams& p, Shared& sh, unsigned char* stages) {
  Ctrl* ctrl = p.ctrl;
  const unsigned int p1_items = static_cast<unsigned int>(p.k) * static_cast<unsigned int>(p.nch);
  uint32_t use = 0;
  bool ok = true;
  unsigned int t = atomicAdd(&ctrl->ticket, 1u);
  while (t < p.total) {
    const unsigned int tn = atomicAdd(&ctrl->ticket, 1u);  // overlaps this chunk
    const unsigned int slot = t / p.slot_items, o = t % p.slot_items;
    Hdr h;
    bool real = false;
    if (o < p1_items) {
      if (static_cast<int>(slot) < p.B) {
        real = true;
        h.kind = kKindStats;
        h.b = static_cast<int>(slot);
        h.i = static_cast<int>(o) / p.nch;
        h.c = static_cast<int>(o) % p.nch;
      }
    } else {
      const int b = static_cast<int>(slot) - p.lag;
      if (b >= 0 && b < p.B) {
        real = true;
        h.b = b;
        h.c = static_cast<int>(o - p1_items);
        int n = 0;
        if (p.k > 0) {
          if (!wait_flag(&p.seq[b].ready, ctrl)) {
            ok = false;
            break;
          }
          // clamped so that no workspace content can steer a read outside
          // the tensors
          n = min(max(__ldcg(&p.seq[b].n), 0), p.k);
        }
        h.i = n;
        if (n < p.k) {
          h.kind = kKindCorrection;
          h.mt = __ldcg(&p.seq[b].mt);
          h.ist = __ldcg(&p.seq[b].ist);
          h.md = __ldcg(&p.seq[b].md);
          h.isd = __ldcg(&p.seq[b].isd);
        } else {
          h.kind = kKindBonus;
        }
      }
    }
    if (real) {
      h.x0 = h.c * p.ch;
      h.len = min(p.ch, p.V - h.x0);
      h.toff = static_cast<long long>(h.b) * p.t_sb + static_cast<long long>(h.i) * p.t_sp + h.x0;
      h.doff = static_cast<long long>(h.b) * p.d_sb + static_cast<long long>(h.i) * p.d_sp + h.x0;
      const int s = use % kStages;
      if (!mbar_wait(&sh.empty[s], ((use / kStages) & 1u) ^ 1u, ctrl)) {
        ok = false;
        break;
      }
      issue_chunk<TT, TD, kTma>(sh, stages + static_cast<size_t>(s) * kStageBytes, s, h, p.tgt,
                                p.drf, p.ch, h.kind != kKindBonus);
      ++use;
    }
    t = tn;
  }
  if (ok) {
    const int s = use % kStages;
    if (mbar_wait(&sh.empty[s], ((use / kStages) & 1u) ^ 1u, ctrl)) {
      sh.hdr[s].kind = kKindEnd;
      mbar_arrive(&sh.full[s]);
    }
    leave_grid(ctrl);
  } else if (kTma) {
    drain_stages(sh, use);
  }
}

template <typename TT, typename TD, bool kTma>
__device__ void stoch_compute(const StochParams& p, Shared& sh, unsigned char* stages, int w,
                              int lane) {
  const int tid = w * 32 + lane;
  for (uint32_t use = 0;; ++use) {
    const int s = use % kStages;
    if (!mbar_wait(&sh.full[s], (use / kStages) & 1u, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd) {
      if (lane == 0) mbar_arrive(&sh.rfull[s]);
      break;
    }
    const unsigned char* ts = stages + static_cast<size_t>(s) * kStageBytes;
    const unsigned char* ds = ts + static_cast<size_t>(p.ch) * Elem<TT>::kBytes;
    float4 r;
    if (h.kind == kKindStats) {
      float m1, s1, m2, s2;
      chunk_stats<TT>(ts, h.nvec_t, p.tgt, h.toff, h.len, p.c2, tid, m1, s1);
      chunk_stats<TD>(ds, h.nvec_d, p.drf, h.doff, h.len, p.c2, tid, m2, s2);
      r = make_float4(m1, s1, m2, s2);
    } else {
      const Draw d{p.key0, p.key1, static_cast<uint32_t>(h.i),
                   static_cast<uint32_t>(h.b) + p.seq_offset,
                   h.kind == kKindCorrection ? kTagCorrection : kTagBonus};
      float bv;
      int bi;
      if (h.kind == kKindCorrection)
        chunk_residual<TT, TD, kTma>(ts, ds, h, p.tgt, p.drf, p.c2, d, tid, bv, bi);
      else
        chunk_bonus<TT, kTma>(ts, h, p.tgt, p.invT, d, tid, bv, bi);
      r = make_float4(bv, __int_as_float(bi), 0.0f, 0.0f);
    }
    if (lane == 0) {
      sh.res[s][w] = r;
      mbar_arrive(&sh.rfull[s]);
    }
  }
}

// Phase-1 finalize of sequence b (one warp): merge chunk statistics per
// position, gather p_i(x_i), q_i(x_i), accept while u_i q < p, publish n.
template <typename TT, typename TD>
__device__ void finalize_accept(const StochParams& p, int b, int lane) {
  const int k = p.k;
  float MT = -INFINITY, ST = 0.0f, MD = -INFINITY, SD = 0.0f;
  bool acc = true;
  if (lane < k) {
    // merge this position's chunk partials, then clear them: every call
    // leaves the workspace zeroed, whatever sizes the next call uses
    float4* part = p.part + (static_cast<size_t>(b) * k + lane) * p.nch;
    for (int c = 0; c < p.nch; ++c) {
      const float4 v = __ldcg(part + c);
      merge_stats(MT, ST, v.x, v.y);
      merge_stats(MD, SD, v.z, v.w);
      part[c] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    const int x = __ldg(p.tokens + static_cast<size_t>(b) * k + lane);
    const bool valid = x >= 0 && x < p.V;
    float pt = 0.0f, qd = 0.0f;
    if (valid) {
      const float lt = load_elem<TT>(
          p.tgt, static_cast<long long>(b) * p.t_sb + static_cast<long long>(lane) * p.t_sp + x);
      const float ld = load_elem<TD>(
          p.drf, static_cast<long long>(b) * p.d_sb + static_cast<long long>(lane) * p.d_sp + x);
      pt = ex2f(fmaf(lt, p.c2, -MT)) / ST;
      qd = ex2f(fmaf(ld, p.c2, -MD)) / SD;
    } else {
      atomicOr(&p.ctrl->flags, kFlagInvalidToken);
    }
    const uint4 w = philox10(
        make_uint4(0u, static_cast<uint32_t>(lane), static_cast<uint32_t>(b) + p.seq_offset,
                   kTagAccept),
        p.key0, p.key1);
    acc = valid && (accept_uniform(w.x) * qd < pt);
    if (p.probs) {
      float* pr = p.probs + (static_cast<size_t>(b) * k + lane) * 2;
      pr[0] = pt;
      pr[1] = qd;
    }
  }
  const unsigned int rej = __ballot_sync(0xffffffffu, !acc);
  const int n = rej ? __ffs(rej) - 1 : k;
  const float smt = __shfl_sync(0xffffffffu, MT, n & 31);
  const float sst = __shfl_sync(0xffffffffu, ST, n & 31);
  const float smd = __shfl_sync(0xffffffffu, MD, n & 31);
  const float ssd = __shfl_sync(0xffffffffu, SD, n & 31);
  int* out = p.out_tokens + static_cast<size_t>(b) * (k + 1);
  for (int i = lane; i <= k; i += 32)
    if (i != n) out[i] = i < n ? __ldg(p.tokens + static_cast<size_t>(b) * k + i) : -1;
  if (lane == 0) {
    p.accepted_len[b] = n;
    SeqRec* r = p.seq + b;
    r->n = n;
    r->mt = smt;
    r->ist = 1.0f / sst;
    r->md = smd;
    r->isd = 1.0f / ssd;
    r->cnt1 = 0u;
    __threadfence();
    st_release_u32(&r->ready, 1u);
  }
}

// Phase-2 finalize of sequence b (one warp): the merged Gumbel-max key gives
// the token at position n.  With no positive residual mass the token is drawn
// from p_n with the same CORRECTION stream (slow path, one warp).
template <typename TT>
__device__ void finalize_sample(const StochParams& p, const Hdr& h, int lane) {
  const int b = h.b, n = h.i, k = p.k;
  unsigned long long key = 0ull;
  if (lane == 0) key = atomicExch(&p.seq[b].key, 0ull);
  key = __shfl_sync(0xffffffffu, key, 0);
  int tok;
  if (key == 0ull) {
    if (lane == 0) atomicOr(&p.ctrl->flags, kFlagResidualFallback);
    const Draw d{p.key0, p.key1, static_cast<uint32_t>(n),
                 static_cast<uint32_t>(b) + p.seq_offset, kTagCorrection};
    const long long off = static_cast<long long>(b) * p.t_sb + static_cast<long long>(n) * p.t_sp;
    float bv = -INFINITY;
    int bi = INT_MAX;
    for (int x = lane; x < p.V; x += 32) {
      const float sc = fmaf(load_elem<TT>(p.tgt, off + x), p.invT,
                            gumbel(word_of(vocab_words(d, static_cast<uint32_t>(x) >> 2), x & 3)));
      if (better(sc, x, bv, bi)) {
        bv = sc;
        bi = x;
      }
    }
    warp_argmax(bv, bi);
    tok = bi;
  } else {
    tok = key_index(key);
  }
  if (lane == 0) {
    p.out_tokens[static_cast<size_t>(b) * (k + 1) + n] = tok;
    p.accepted_len[b] = n;
    SeqRec* r = p.seq + b;
    r->n = 0;
    r->mt = r->ist = r->md = r->isd = 0.0f;
    r->cnt2 = 0u;
    r->ready = 0u;
  }
}

template <typename TT, typename TD>
__device__ void stoch_epilogue(const StochParams& p, Shared& sh, int lane) {
  for (uint32_t use = 0;; ++use) {
    const int s = use % kStages;
    if (!mbar_wait(&sh.rfull[s], (use / kStages) & 1u, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd) break;
    float4 r = lane < kComputeWarps ? sh.res[s][lane]
                                    : make_float4(-INFINITY, __int_as_float(INT_MAX), 0.f, 0.f);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.empty[s]);
    bool last = false;
    if (h.kind == kKindStats) {
      if (lane >= kComputeWarps) r = make_float4(-INFINITY, 0.0f, -INFINITY, 0.0f);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float a = __shfl_xor_sync(0xffffffffu, r.x, o);
        const float b = __shfl_xor_sync(0xffffffffu, r.y, o);
        const float c = __shfl_xor_sync(0xffffffffu, r.z, o);
        const float d = __shfl_xor_sync(0xffffffffu, r.w, o);
        merge_stats(r.x, r.y, a, b);
        merge_stats(r.z, r.w, c, d);
      }
      if (lane == 0) {
        p.part[(static_cast<size_t>(h.b) * p.k + h.i) * p.nch + h.c] = r;
        __threadfence();
        last = atomicAdd(&p.seq[h.b].cnt1, 1u) ==
               static_cast<unsigned int>(p.k) * static_cast<unsigned int>(p.nch) - 1u;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        finalize_accept<TT, TD>(p, h.b, lane);
      }
    } else {
      float v = r.x;
      int i = __float_as_int(r.y);
      warp_argmax(v, i);
      if (lane == 0) {
        if (i != INT_MAX) atomicMax(&p.seq[h.b].key, make_key(v, i));
        __threadfence();
        last = atomicAdd(&p.seq[h.b].cnt2, 1u) == static_cast<unsigned int>(p.nch) - 1u;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence();
        finalize_sample<TT>(p, h, lane);
      }
    }
  }
}

template <typename TT, typename TD, bool kTma>
__global__ void __launch_bounds__(kThreads, 1)
    stochastic_verify_kernel(const __grid_constant__ StochParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared& sh = *reinterpret_cast<Shared*>(smem_raw);
  unsigned char* stages = smem_raw + kSharedHead;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
      mbar_init(&sh.rfull[s], kComputeWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) stoch_producer<TT, TD, kTma>(p, sh, stages);
  } else if (warp <= kComputeWarps) {
    stoch_compute<TT, TD, kTma>(p, sh, stages, warp - 1, lane);
  } else {
    stoch_epilogue<TT, TD>(p, sh, lane);
  }
}

// ================================================================ argmax

template <typename TT, bool kTma>
__device__ void argmax_producer(const ArgmaxParams& p, Shared& sh, unsigned char* stages) {
  Ctrl* ctrl = p.ctrl;
  const unsigned int R = static_cast<unsigned int>(p.G) * static_cast<unsigned int>(p.k + 1);
  const unsigned int per_seq = R * static_cast<unsigned int>(p.nch);
  uint32_t use = 0;
  bool ok = true;
  unsigned int t = atomicAdd(&ctrl->ticket, 1u);
  while (t < p.total) {
    const unsigned int tn = atomicAdd(&ctrl->ticket, 1u);
    Hdr h;
    h.kind = kKindArgmax;
    h.b = static_cast<int>(t / per_seq);
    const unsigned int rem = t % per_seq;
    h.i = static_cast<int>(rem / p.nch);
    h.c = static_cast<int>(rem % p.nch);
    const int g = h.i / (p.k + 1), pos = h.i % (p.k + 1);
    h.x0 = h.c * p.ch;
    h.len = min(p.ch, p.V - h.x0);
    h.toff = static_cast<long long>(h.b) * p.sb + static_cast<long long>(g) * p.sg +
             static_cast<long long>(pos) * p.sp + h.x0;
    h.doff = 0;
    const int s = use % kStages;
    if (!mbar_wait(&sh.empty[s], ((use / kStages) & 1u) ^ 1u, ctrl)) {
      ok = false;
      break;
    }
    issue_chunk<TT, TT, kTma>(sh, stages + static_cast<size_t>(s) * kStageBytes, s, h, p.tgt,
                              nullptr, p.ch, false);
    ++use;
    t = tn;
  }
  if (ok) {
    const int s = use % kStages;
    if (mbar_wait(&sh.empty[s], ((use / kStages) & 1u) ^ 1u, ctrl)) {
      sh.hdr[s].kind = kKindEnd;
      mbar_arrive(&sh.full[s]);
    }
    leave_grid(ctrl);
  } else if (kTma) {
    drain_stages(sh, use);
  }
}

template <typename TT>
__device__ void argmax_compute(const ArgmaxParams& p, Shared& sh, unsigned char* stages, int w,
                               int lane) {
  const int tid = w * 32 + lane;
  for (uint32_t use = 0;; ++use) {
    const int s = use % kStages;
    if (!mbar_wait(&sh.full[s], (use / kStages) & 1u, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd) {
      if (lane == 0) mbar_arrive(&sh.rfull[s]);
      break;
    }
    float bv;
    int bi;
    chunk_argmax<TT>(stages + static_cast<size_t>(s) * kStageBytes, h, p.tgt, tid, bv, bi);
    if (lane == 0) {
      sh.res[s][w] = make_float4(bv, __int_as_float(bi), 0.0f, 0.0f);
      mbar_arrive(&sh.rfull[s]);
    }
  }
}

// Finalize of sequence b (one warp): per branch, the accepted length is the
// first position whose draft differs from the row argmax (ballot); the
// longest branch (lowest g on a tie) is committed.
__device__ void finalize_argmax(const ArgmaxParams& p, int b, int lane) {
  const int k = p.k, G = p.G;
  unsigned long long* keys = p.rowkey + static_cast<size_t>(b) * G * (k + 1);
  int best_n = -1, best_g = 0, best_next = -1;
  for (int g = 0; g < G; ++g) {
    unsigned long long* gk = keys + static_cast<size_t>(g) * (k + 1);
    int a = -1, a32 = -1;
    if (lane <= k) a = key_index(atomicExch(gk + lane, 0ull));
    if (k == 32 && lane == 0) a32 = key_index(atomicExch(gk + 32, 0ull));
    const int* cand = p.tokens + (static_cast<size_t>(b) * G + g) * k;
    const bool miss = lane < k && __ldg(cand + lane) != a;
    const unsigned int mm = __ballot_sync(0xffffffffu, miss);
    const int n = mm ? __ffs(mm) - 1 : k;
    const int an = __shfl_sync(0xffffffffu, a, n & 31);
    const int a32b = __shfl_sync(0xffffffffu, a32, 0);
    if (n > best_n) {
      best_n = n;
      best_g = g;
      best_next = (n == 32) ? a32b : an;
    }
  }
  const int* cand = p.tokens + (static_cast<size_t>(b) * G + best_g) * k;
  int* out = p.out_tokens + static_cast<size_t>(b) * (k + 1);
  for (int i = lane; i <= k; i += 32)
    out[i] = i < best_n ? __ldg(cand + i) : (i == best_n ? best_next : -1);
  if (lane == 0) {
    p.accepted_len[b] = best_n;
    if (p.best_g) p.best_g[b] = best_g;
    p.seq[b].cnt1 = 0u;
  }
}

__device__ void argmax_epilogue(const ArgmaxParams& p, Shared& sh, int lane) {
  const unsigned int R = static_cast<unsigned int>(p.G) * static_cast<unsigned int>(p.k + 1);
  for (uint32_t use = 0;; ++use) {
    const int s = use % kStages;
    if (!mbar_wait(&sh.rfull[s], (use / kStages) & 1u, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd) break;
    float v = -INFINITY;
    int i = INT_MAX;
    if (lane < kComputeWarps) {
      const float4 r = sh.res[s][lane];
      v = r.x;
      i = __float_as_int(r.y);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.empty[s]);
    warp_argmax(v, i);
    bool last = false;
    if (lane == 0) {
      atomicMax(p.rowkey + static_cast<size_t>(h.b) * R + h.i, make_key(v, i));
      __threadfence();
      last = atomicAdd(&p.seq[h.b].cnt1, 1u) == R * static_cast<unsigned int>(p.nch) - 1u;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __threadfence();
      finalize_argmax(p, h.b, lane);
    }
  }
}

template <typename TT, bool kTma>
__global__ void __launch_bounds__(kThreads, 1)
    argmax_verify_kernel(const __grid_constant__ ArgmaxParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Shared& sh = *reinterpret_cast<Shared*>(smem_raw);
  unsigned char* stages = smem_raw + kSharedHead;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.empty[s], 1);
      mbar_init(&sh.rfull[s], kComputeWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) argmax_producer<TT, kTma>(p, sh, stages);
  } else if (warp <= kComputeWarps) {
    argmax_compute<TT>(p, sh, stages, warp - 1, lane);
  } else {
    argmax_epilogue(p, sh, lane);
  }
}

// ================================================================ philox

__global__ void philox_kernel(const uint4* __restrict__ ctr, long long n, uint32_t k0,
                              uint32_t k1, uint4* __restrict__ out) {
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < n;
       j += static_cast<long long>(gridDim.x) * blockDim.x)
    out[j] = philox10(ctr[j], k0, k1);
}

// ============================================================== launchers

// The shared-memory opt-in is per function and device; setting it again is
// harmless, so each kernel instantiation keeps a per-device "done" bit.
template <typename K>
static cudaError_t prepare(K kernel, size_t smem, bool (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

template <typename TT, typename TD, bool kTma>
static cudaError_t launch_stoch_t(const StochParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool done[64] = {};
  auto kernel = stochastic_verify_kernel<TT, TD, kTma>;
  cudaError_t e = prepare(kernel, smem, done);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename TT, typename TD>
static cudaError_t launch_stoch_tma(const StochParams& p, bool tma, int grid, size_t smem,
                                    cudaStream_t st) {
  return tma ? launch_stoch_t<TT, TD, true>(p, grid, smem, st)
             : launch_stoch_t<TT, TD, false>(p, grid, smem, st);
}

cudaError_t launch_stochastic(const StochParams& p, int t_dtype, int d_dtype, bool tma, int grid,
                              size_t smem, cudaStream_t st) {
  if (t_dtype == 1 && d_dtype == 1) return launch_stoch_tma<uint16_t, uint16_t>(p, tma, grid, smem, st);
  if (t_dtype == 1 && d_dtype == 0) return launch_stoch_tma<uint16_t, float>(p, tma, grid, smem, st);
  if (t_dtype == 0 && d_dtype == 1) return launch_stoch_tma<float, uint16_t>(p, tma, grid, smem, st);
  return launch_stoch_tma<float, float>(p, tma, grid, smem, st);
}

template <typename TT, bool kTma>
static cudaError_t launch_argmax_t(const ArgmaxParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool done[64] = {};
  auto kernel = argmax_verify_kernel<TT, kTma>;
  cudaError_t e = prepare(kernel, smem, done);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_argmax(const ArgmaxParams& p, int t_dtype, bool tma, int grid, size_t smem,
                          cudaStream_t st) {
  if (t_dtype == 1)
    return tma ? launch_argmax_t<uint16_t, true>(p, grid, smem, st)
               : launch_argmax_t<uint16_t, false>(p, grid, smem, st);
  return tma ? launch_argmax_t<float, true>(p, grid, smem, st)
             : launch_argmax_t<float, false>(p, grid, smem, st);
}

cudaError_t launch_philox(const uint4* ctr, long long n, unsigned int key0, unsigned int key1,
                          uint4* out, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const long long blocks = (n + 255) / 256;
  const int grid = static_cast<int>(blocks < 4096 ? blocks : 4096);
  philox_kernel<<<grid, 256, 0, st>>>(ctr, n, key0, key1, out);
  return cudaGetLastError();
}

}  // namespace sv
