// sv_kernels.cu -- persistent verify kernels for sm_100a.
//
// One CTA per SM runs until the work tickets run out.  A ticket names one
// chunk of one row (or row pair): the vocabulary of every row is split into
// `nch` chunks, so each (sequence, position) row is reduced by many CTAs.
//
//   warps 0, 1       producers (lane 0): take tickets (atomicAdd, one grab
//                    ahead) and stream each chunk into a 4-stage shared-
//                    memory ring with 1-D bulk copies (TMA, cp.async.bulk)
//                    that complete on an mbarrier.  In the stochastic kernel
//                    each producer feeds its own compute group's two stages;
//                    the argmax kernels use warp 0 alone, alternating groups.
//                    A chunk whose sequence is not ready yet (phase 2 below)
//                    is set aside in a short queue and issued once it is, so
//                    the ring keeps flowing.
//   warps 2..17      compute, two groups of 8: reduce the chunk held in shared
//                    memory (softmax statistics, Gumbel-max, or argmax) to one
//                    record per warp.
//   last 2 warps     epilogues, one per compute group: merge the warp records, publish the
//                    chunk's partial with one 64-bit store and counts it with
//                    a relaxed atomicAdd on its row's counter.  A published
//                    partial is never zero, so the value is its own "ready"
//                    flag and no fence is needed.  The counter's old value is
//                    checked one chunk later (or at once when no chunk is
//                    waiting), so its round trip overlaps work.  Merging is
//                    two-level: the CTA that completes a row merges the row's
//                    chunk partials (one lane per chunk, one round trip) into
//                    a row record and counts the row on the sequence; the CTA
//                    that completes a sequence finalizes it from its row
//                    records.  Every slot and counter is cleared after use.
//
// Stochastic verify ("Accelerating Sonar through speculation", section
// "Draft-Target": acceptance compares the full draft and target
// distributions; the target's logits after the accepted prefix are sampled)
// runs in two phases on the same ticket counter:
//   phase 1  chunks of row pairs (target i, draft i), i < k: per-chunk
//            softmax statistics (max and sum of 2^(x log2(e)/T - max)).  The
//            finalizer merges them, gathers p_i(x_i) and q_i(x_i), draws u_i
//            (Philox, tag ACCEPT), finds the first rejection n with a warp
//            ballot and publishes n (release store of a ready flag).
//   phase 2  the `nch` chunks of the row that gives the next token: the row
//            pair n (correction: Gumbel-max over ln max(0, p_n - q_n)) or
//            target row k (bonus: Gumbel-max over l_k / T).  They sit `lag`
//            sequences after their phase-1 chunks in ticket order, so the
//            pair is usually still in L2 and the producer rarely waits.
// Target row k is read only for sequences that accept all k drafts.
//
// Greedy and multi-candidate verify ("Lookahead decoding" news piece,
// section "Lookahead decoding breaks the order dependency") are one phase:
// per-chunk argmax keys; the finalizer takes each row's maximum key, compares
// every branch's drafts with its row argmaxes (warp ballot) and commits the
// longest branch.
//
// Every wait is bounded (kWaitLimitNs); on expiry the kernel raises
// kFlagTimeout, every role leaves its loop, and the producer waits for its
// bulk copies in flight before the CTA exits.  A producer only waits for a
// sequence whose phase-1 chunks all carry smaller tickets than the one it
// waits with; those are held by running CTAs, which issue their fresh
// tickets in order and never hold a set-aside ticket smaller than a fresh
// one, and an epilogue settles every arrival before it blocks again, so
// every wait ends.
#include <climits>

#include "sv_device.cuh"

namespace sv {

enum : int {
  kKindEnd = 0,
  kKindStats = 1,
  kKindCorrection = 2,
  kKindBonus = 3,
  kKindArgmax = 4,
  kKindRowDone = 5  // no data: the producer retired the last chunks of row (b, i) unread
};

// Argmax tickets per atomicAdd (the next grab's atomic is always in
// flight): argmax chunks are uniform work, so larger grabs save atomics.
// Stochastic tickets are taken one at a time, which balances the uneven
// phase-1 and phase-2 chunks best.
#ifndef SV_GRAB_ARGMAX
#define SV_GRAB_ARGMAX 8
#endif
constexpr unsigned int kGrabArgmax = SV_GRAB_ARGMAX;
// Producers of the argmax kernels: 1 (warp 0 alternates the two groups'
// stages) or 2 (one per compute group, each filling its own two stages).
#ifndef SV_ARGMAX_PRODUCERS
#define SV_ARGMAX_PRODUCERS 1
#endif
constexpr int kArgmaxProducers = SV_ARGMAX_PRODUCERS;
static_assert(kArgmaxProducers == 1 || kArgmaxProducers == kComputeGroups, "1 or one per group");
constexpr unsigned long long kNoCandidate = 1ull;  // phase-2 key: no positive residual
// Argmax chunk key of a chunk retired unread: below every real key (whose
// high word is at least orderable(-inf) > 0), and never zero.
constexpr unsigned long long kSkippedKey = 1ull;

struct Hdr {
  int kind;
  int b;       // sequence
  int i;       // position (stochastic) or row within the sequence (argmax)
  int c;       // chunk
  int x0;      // first vocabulary entry of the chunk
  int len;     // entries in the chunk
  int nvec_t;  // full 16-byte target vectors in shared memory
  int nvec_d;  // full 16-byte draft vectors in shared memory
  long long toff;          // element offset of entry x0 in the target
  long long doff;          // element offset of entry x0 in the draft
  int slot;                // phase 2: the sequence's ready-list entry
};

struct Shared {
  uint64_t full[kStages];   // producer -> compute (bulk-copy bytes)
  uint64_t empty[kStages];  // epilogue -> producer (slot free)
  uint64_t rfull[kStages];  // compute -> epilogue (warp records written)
  Hdr hdr[kStages];
  float4 res[kStages][kGroupWarps];
  float4 rstat[kStages];  // correction: row-n (m_t, 1/s_t, m_d, 1/s_d), bulk-copied
};

constexpr size_t kSharedHead = (sizeof(Shared) + 127) / 128 * 128;

size_t kernel_smem_bytes() { return kSharedHead + static_cast<size_t>(kStages) * kStageBytes; }

// ----------------------------------------------------------- publish/poll

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Wait (bounded) until a published partial appears; 0 on timeout/abort.
__device__ __forceinline__ unsigned long long poll_u64(const unsigned long long* p, Ctrl* ctrl) {
  unsigned long long v = ld_relaxed_u64(p);
  if (v) return v;
  const unsigned long long t0 = global_ns();
  for (unsigned int spin = 1;; ++spin) {
    v = ld_relaxed_u64(p);
    if (v) return v;
    if ((spin & 63u) == 0u) {
      if (aborted(ctrl)) return 0ull;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicOr(&ctrl->flags, kFlagTimeout);
        return 0ull;
      }
    }
  }
}

// (max, sum) packed in 64 bits.  sum >= 1 for any chunk with a finite max
// and max = -inf otherwise, so a published pair is never all-zero bits.
__device__ __forceinline__ unsigned long long pack_stats(float m, float s) {
  return (static_cast<unsigned long long>(__float_as_uint(s)) << 32) | __float_as_uint(m);
}
__device__ __forceinline__ void unpack_stats(unsigned long long v, float& m, float& s) {
  m = __uint_as_float(static_cast<uint32_t>(v & 0xffffffffull));
  s = __uint_as_float(static_cast<uint32_t>(v >> 32));
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// ------------------------------------------------------------------ waits

// Waits (bounded) for a nonzero flag; returns its value, or 0 on abort or
// timeout.  Acquire: the flag's writer's earlier stores are visible after.
__device__ __forceinline__ unsigned int wait_flag(const unsigned int* flag, Ctrl* ctrl) {
  unsigned int v = ld_acquire_u32(flag);
  if (v) return v;
  const unsigned long long t0 = global_ns();
  for (unsigned int spin = 1;; ++spin) {
    __nanosleep(32);
    v = ld_acquire_u32(flag);
    if (v) return v;
    if ((spin & 63u) == 0u) {
      if (aborted(ctrl)) return 0u;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicOr(&ctrl->flags, kFlagTimeout);
        return 0u;
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

__device__ __forceinline__ unsigned int udiv(unsigned int n, const UDiv& u) {
  return u.m ? __umulhi(n, u.m) >> u.shift : n;
}

__device__ __forceinline__ void leave_grid(Ctrl* ctrl, unsigned int producers_per_cta) {
  // The last producer to take its final ticket rewinds the ticket counter.
  if (atomicAdd(&ctrl->exits, 1u) == gridDim.x * producers_per_cta - 1) {
    atomicExch(&ctrl->ticket, 0u);
    atomicExch(&ctrl->exits, 0u);
  }
}

// Fill stage `s` with the chunk described by `h` (bulk copies of the full
// 16-byte vectors; the ragged end is read by the compute warps directly).
// `stat` (nullable, 16-byte aligned, global): a row-statistics record that
// goes to sh.rstat[s] with the chunk.
template <typename TT, typename TD, bool kTma>
__device__ __forceinline__ void issue_chunk(Shared& sh, unsigned char* stage, int s, Hdr& h,
                                            const void* tgt, const void* drf, int ch,
                                            bool with_draft, const float4* stat) {
  h.nvec_t = kTma ? (h.len * Elem<TT>::kBytes) / 16 : 0;
  h.nvec_d = (kTma && with_draft) ? (h.len * Elem<TD>::kBytes) / 16 : 0;
  sh.hdr[s] = h;
  if (kTma) {
    const uint32_t bt = static_cast<uint32_t>(h.nvec_t) * 16u;
    const uint32_t bd = static_cast<uint32_t>(h.nvec_d) * 16u;
    mbar_arrive_expect_tx(&sh.full[s], bt + bd + (stat ? 16u : 0u));
    if (bt) bulk_load(stage, reinterpret_cast<const TT*>(tgt) + h.toff, bt, &sh.full[s]);
    if (bd)
      bulk_load(stage + static_cast<size_t>(ch) * Elem<TT>::kBytes,
                reinterpret_cast<const TD*>(drf) + h.doff, bd, &sh.full[s]);
    if (stat) bulk_load(&sh.rstat[s], stat, 16u, &sh.full[s]);
  } else {
    if (stat) sh.rstat[s] = __ldcg(stat);
    mbar_arrive(&sh.full[s]);
  }
}

// --- per-group rings (stochastic kernel) -----------------------------------
// Compute group g owns stages g and g + 2 and has its own producer; its j-th
// use is stage g + 2 (j % 2), phase (j / 2) & 1 -- the order in which its
// producer, compute warps and epilogue warp walk them.  Each group is its own
// pipeline, so a group busy with a long chunk does not hold the other back.
constexpr int kGroupStages = kStages / kComputeGroups;
static_assert(kGroupStages * kComputeGroups == kStages, "stages split evenly over groups");

__device__ __forceinline__ int group_stage(int g, uint32_t j) {
  return g + kComputeGroups * static_cast<int>(j % kGroupStages);
}
__device__ __forceinline__ uint32_t group_phase(uint32_t j) { return (j / kGroupStages) & 1u; }

// One end marker into group g's next stage.
__device__ __forceinline__ void push_group_end(Shared& sh, int g, uint32_t used, Ctrl* ctrl) {
  const int s = group_stage(g, used);
  if (!mbar_wait(&sh.empty[s], group_phase(used) ^ 1u, ctrl)) return;
  sh.hdr[s].kind = kKindEnd;
  mbar_arrive(&sh.full[s]);
}

// After an abort: wait (bounded) until the last bulk copy issued into each of
// group g's stages has landed.
__device__ void drain_group_stages(Shared& sh, int g, uint32_t used) {
  for (uint32_t r = 0; r < static_cast<uint32_t>(kGroupStages) && r < used; ++r) {
    const uint32_t last = r + ((used - 1 - r) / kGroupStages) * kGroupStages;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(&sh.full[group_stage(g, r)], group_phase(last))) {
      if (global_ns() - t0 > 100000000ull) break;
    }
  }
}

// Push one end marker per compute group into the next stages.
__device__ __forceinline__ void push_end(Shared& sh, uint32_t use, Ctrl* ctrl) {
  for (int g = 0; g < kComputeGroups; ++g, ++use) {
    const int s = use % kStages;
    if (!mbar_wait(&sh.empty[s], ((use / kStages) & 1u) ^ 1u, ctrl)) return;
    sh.hdr[s].kind = kKindEnd;
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
  float mc = -INFINITY, s = 0.0f;
  if (m != -INFINITY) {
    mc = m * c2;
    float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 2
    for (int v = tid; v < nvec; v += kComputeThreads) {
      float f[EPV];
      unpack(sv[v], f);
#pragma unroll
      for (int j = 0; j < EPV; j += 2) {
        s0 += ex2f(fmaf(f[j], c2, -mc));
        s1 += ex2f(fmaf(f[j + 1], c2, -mc));
      }
    }
    for (int e = nvec * EPV + tid; e < len; e += kComputeThreads)
      s0 += ex2f(fmaf(load_elem<T>(g, goff + e), c2, -mc));
    s = warp_sum(s0 + s1);
  }
  m_out = mc;
  s_out = s;
}

// --- register-resident reductions (bulk-copy path) -----------------------
// Every thread loads all of its 16-byte vectors of the chunk at once
// (vectors tid, tid + 512, ...), padding with -inf, so each warp has a
// whole chunk's worth of independent loads, exps and maxima in flight and
// no reduction sits between the max and the sum.

// Most vectors one thread holds for a tensor of element type T in a chunk of
// a `bytes` budget shared with a partner tensor of element size `partner`
// bytes (0: the tensor has the chunk to itself); a full chunk gives every
// thread exactly this many.
template <typename T, int partner, int bytes>
__host__ __device__ constexpr int max_vecs() {
  return (full_chunk_entries(bytes, Elem<T>::kBytes + partner,
                             partner > 0 && partner < Elem<T>::kBytes ? partner : Elem<T>::kBytes) *
              Elem<T>::kBytes / 16 +
          kComputeThreads - 1) /
         kComputeThreads;
}

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

template <typename T, int N>
__device__ __forceinline__ void load_vecs(const unsigned char* smem, int nvec, int tid,
                                          uint4 (&v)[N]) {
  const uint4* sv = reinterpret_cast<const uint4*>(smem);
  if (nvec == N * kComputeThreads) {  // a full chunk (uniform): no padding
#pragma unroll
    for (int j = 0; j < N; ++j) v[j] = sv[tid + j * kComputeThreads];
  } else {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int idx = tid + j * kComputeThreads;
      v[j] = idx < nvec ? sv[idx] : neg_inf_vec<T>();
    }
  }
}

// One pair in kPolyEvery of the register-resident exponentials runs on the FMA
// pipe (ex2_poly_x2) instead of the special-function unit, which the
// statistics otherwise saturate.
#ifndef SV_POLY_EVERY
#define SV_POLY_EVERY 8
#endif
constexpr int kPolyEvery = SV_POLY_EVERY;

// Warp merge of per-thread (m, s) pairs of two tensors: the maxima first,
// then one rescale per thread and a plain sum.
__device__ __forceinline__ float4 warp_stats2(float4 r) {
  const float Mt = warp_max(r.x), Md = warp_max(r.z);
  float st = Mt == -INFINITY ? 0.0f : r.y * ex2f(r.x - Mt);
  float sd = Md == -INFINITY ? 0.0f : r.w * ex2f(r.z - Md);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    st += __shfl_xor_sync(0xffffffffu, st, o);
    sd += __shfl_xor_sync(0xffffffffu, sd, o);
  }
  return make_float4(Mt, st, Md, sd);
}

// Largest element of N vectors (the -inf padding included).
template <typename T, int N>
__device__ __forceinline__ float vecs_max(const uint4 (&v)[N]) {
  if constexpr (Elem<T>::kBytes == 2) {
    // bf16: a running packed maximum, one max.bf16x2 per two elements
    uint32_t m = 0xff80ff80u;
#pragma unroll
    for (int j = 0; j < N; ++j) m = bmax2(m, bmax2(bmax2(v[j].x, v[j].y), bmax2(v[j].z, v[j].w)));
    return fmaxf(bf16_lo(m), bf16_hi(m));
  } else {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < N; ++j) {
      m = fmax3(m, __uint_as_float(v[j].x), __uint_as_float(v[j].y));
      m = fmax3(m, __uint_as_float(v[j].z), __uint_as_float(v[j].w));
    }
    return m;
  }
}

// Thread-local (m, s): m = max * c2 (log2 units), s = sum 2^(x c2 - m)
// over the thread's vectors plus its share of the ragged end in global
// memory (entries [tail0, len)).
template <typename T, int N>
__device__ __forceinline__ void thread_stats(const uint4 (&v)[N], const void* g, long long goff,
                                             int tail0, int len, float c2, int tid, float& m_out,
                                             float& s_out) {
  constexpr int EPV = Elem<T>::kPerVec;
  float m = vecs_max<T>(v);
  float tail = -INFINITY;
  const int e = tail0 + tid;  // the ragged end is shorter than one vector
  if (e < len) tail = load_elem<T>(g, goff + e);
  m = fmaxf(m, tail);
  float s = 0.0f, mc = -INFINITY;
  if (m != -INFINITY) {
    mc = m * c2;
    // pairs of entries: one f32x2 FMA for the exponents, one f32x2 add
    const unsigned long long cc = pack2(c2, c2), mm = pack2(-mc, -mc);
    unsigned long long acc0 = 0ull, acc1 = 0ull;  // +0.0f pairs
#pragma unroll
    for (int j = 0; j < N; ++j) {
      float f[EPV];
      unpack(v[j], f);
#pragma unroll
      for (int q = 0; q < EPV; q += 2) {
        float a, b;
        unpack2(fma2(pack2(f[q], f[q + 1]), cc, mm), a, b);
        const unsigned long long e = ((j * EPV + q) / 2) % kPolyEvery == kPolyEvery - 1
                                         ? ex2_poly_x2(a, b)
                                         : pack2(ex2f(a), ex2f(b));
        if ((q & 2) == 0) acc0 = add2(acc0, e);
        else acc1 = add2(acc1, e);
      }
    }
    float a0, a1, b0, b1;
    unpack2(acc0, a0, a1);
    unpack2(acc1, b0, b1);
    s = ((a0 + a1) + (b0 + b1)) + ex2f(fmaf(tail, c2, -mc));
  }
  m_out = mc;
  s_out = s;
}

// Softmax statistics of a (target, draft) chunk pair, merged over the warp.
template <typename TT, typename TD>
__device__ __forceinline__ float4 chunk_stats_pair(const unsigned char* ts,
                                                   const unsigned char* ds, const Hdr& h,
                                                   const void* tgt, const void* drf, float c2,
                                                   int tid) {
  constexpr int NT = max_vecs<TT, Elem<TD>::kBytes, kStochChunkBytes>();
  constexpr int ND = max_vecs<TD, Elem<TT>::kBytes, kStochChunkBytes>();
  uint4 vt[NT], vd[ND];
  load_vecs<TT>(ts, h.nvec_t, tid, vt);
  load_vecs<TD>(ds, h.nvec_d, tid, vd);
  float4 r;
  thread_stats<TT>(vt, tgt, h.toff, h.nvec_t * Elem<TT>::kPerVec, h.len, c2, tid, r.x, r.y);
  thread_stats<TD>(vd, drf, h.doff, h.nvec_d * Elem<TD>::kPerVec, h.len, c2, tid, r.z, r.w);
  return warp_stats2(r);
}

// Argmax (first maximum) of a chunk held in shared memory, merged over the
// warp.
template <typename T>
__device__ __forceinline__ void chunk_argmax_regs(const unsigned char* smem, const Hdr& h,
                                                  const void* g, int tid, float& bv, int& bi) {
  constexpr int EPV = Elem<T>::kPerVec;
  constexpr int N = max_vecs<T, 0, kArgmaxChunkBytes>();
  uint4 v[N];
  load_vecs<T>(smem, h.nvec_t, tid, v);
  // one pass: the first vector holding the thread's maximum, kept whole
  float best = -INFINITY;
  int bj = -1;
  uint4 bvec = v[0];
  const bool full = h.nvec_t == N * kComputeThreads;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float m = vec_max<T>(v[j]);
    const bool take = (full || tid + j * kComputeThreads < h.nvec_t) && (bj < 0 || m > best);
    best = take ? m : best;
    bj = take ? j : bj;
    bvec = take ? v[j] : bvec;
  }
  int idx = INT_MAX;
  if (bj >= 0) {
    float f[EPV];
    unpack(bvec, f);
    const int x = h.x0 + (tid + bj * kComputeThreads) * EPV;
#pragma unroll
    for (int q = EPV - 1; q >= 0; --q)
      if (f[q] == best) idx = x + q;
  }
  const int e = h.nvec_t * EPV + tid;  // the ragged end is shorter than one vector
  if (e < h.len) {
    const float t = load_elem<T>(g, h.toff + e);
    if (better(t, h.x0 + e, best, idx)) {
      best = t;
      idx = h.x0 + e;
    }
  }
  warp_argmax(best, idx);
  bv = best;
  bi = idx;
}

// Argmax and softmax statistics of one chunk from the same registers
// (threshold acceptance): returns (max value, its index as float bits,
// m = max * c2, s = sum 2^(x c2 - m)), merged over the warp.
template <typename T>
__device__ __forceinline__ float4 chunk_argmax_stats_regs(const unsigned char* smem, const Hdr& h,
                                                          const void* g, float c2, int tid,
                                                          Shared& sh, int s, int lane) {
  constexpr int EPV = Elem<T>::kPerVec;
  constexpr int N = max_vecs<T, 0, kArgmaxChunkBytes>();
  uint4 v[N];
  load_vecs<T>(smem, h.nvec_t, tid, v);
  float best = -INFINITY;
  int bj = -1;
  uint4 bvec = v[0];
  const bool full = h.nvec_t == N * kComputeThreads;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float m = vec_max<T>(v[j]);
    const bool take = (full || tid + j * kComputeThreads < h.nvec_t) && (bj < 0 || m > best);
    best = take ? m : best;
    bj = take ? j : bj;
    bvec = take ? v[j] : bvec;
  }
  int idx = INT_MAX;
  if (bj >= 0) {
    float f[EPV];
    unpack(bvec, f);
    const int x = h.x0 + (tid + bj * kComputeThreads) * EPV;
#pragma unroll
    for (int q = EPV - 1; q >= 0; --q)
      if (f[q] == best) idx = x + q;
  }
  const int e = h.nvec_t * EPV + tid;  // the ragged end is shorter than one vector
  if (e < h.len) {
    const float t = load_elem<T>(g, h.toff + e);
    if (better(t, h.x0 + e, best, idx)) {
      best = t;
      idx = h.x0 + e;
    }
  }
  float m, sum;
  thread_stats<T>(v, g, h.toff, h.nvec_t * EPV, h.len, c2, tid, m, sum);
  warp_argmax(best, idx);
  const float4 st = warp_stats2(make_float4(m, sum, -INFINITY, 0.0f));
  return make_float4(best, __int_as_float(idx), st.x, st.y);
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


// Round keys computed once per chunk (SV_PHILOX_ROUND_KEYS) or per draw.
#ifndef SV_PHILOX_ROUND_KEYS
#define SV_PHILOX_ROUND_KEYS 0
#endif
#if SV_PHILOX_ROUND_KEYS
struct ChunkDraw {
  PhiloxKeys k;
  uint32_t pos, seq, tag;
};
__device__ __forceinline__ ChunkDraw chunk_draw(const Draw& d) {
  return ChunkDraw{philox_keys(d.key0, d.key1), d.pos, d.seq, d.tag};
}
__device__ __forceinline__ uint4 vocab_words(const ChunkDraw& d, uint32_t c0) {
  return philox10(make_uint4(c0, d.pos, d.seq, d.tag), d.k);
}
#else
__device__ __forceinline__ const Draw& chunk_draw(const Draw& d) { return d; }
#endif

// Residual of the correction race, rescaled by the row's target sum s_t:
//   r'(x) = 2^(l_t(x) c2 - m_t) - 2^(l_d(x) c2 - m_d + o),   o = lg2(1/s_d) - lg2(1/s_t),
// which is s_t (p(x) - q(x)).  s_t is one positive constant per row, so the
// winner of the race over r'/E is the winner over (p - q)/E.  Identical
// target and draft rows have equal statistics, o = 0 exactly, and r' = 0
// exactly.
struct ResidualTerms {
  float c2, mt, mdo;  // c2, m_t, m_d - o
};
__device__ __forceinline__ ResidualTerms residual_terms(float c2, const float4& st) {
  return ResidualTerms{c2, st.x, st.z - (lg2f(st.w) - lg2f(st.y))};
}
__device__ __forceinline__ float residual(float lt, float ld, const ResidualTerms& rt) {
  return ex2f(fmaf(lt, rt.c2, -rt.mt)) - ex2f(fmaf(ld, rt.c2, -rt.mdo));
}

// The same for eight entries, two at a time (f32x2 exponents and difference).
__device__ __forceinline__ void residual8(const float (&lt)[8], const float (&ld)[8],
                                          const ResidualTerms& rt, float (&r)[8]) {
  const unsigned long long cc = splat2(rt.c2);
  const unsigned long long mt = splat2(-rt.mt), md = splat2(-rt.mdo);
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float a0, a1, b0, b1;
    unpack2(fma2(pack2(lt[e], lt[e + 1]), cc, mt), a0, a1);
    unpack2(fma2(pack2(ld[e], ld[e + 1]), cc, md), b0, b1);
    unpack2(sub2(pack2(ex2f(a0), ex2f(a1)), pack2(ex2f(b0), ex2f(b1))), r[e], r[e + 1]);
  }
}

// Exponential race: argmax_x r(x)/E(x) with E = -ln u'(x) is the Gumbel-max
// argmax_x ln r(x) + g(x).  Keeps the best (r, e, x) of one thread, with e the
// draw in negative log2 units (e = -E / ln 2 < 0).  r/E > b.r/b.E is
// r b.e < b.r e; a candidate with r <= 0 never passes it (its left side is
// >= 0 > the right side once b.r > 0, and -r < -0 fails for the initial
// b = (0, -1)), and the first x is kept on a tie.
struct Race {
  float r, e;
  int x;
};

__device__ __forceinline__ void race_push(Race& b, float r, float e, int x) {
  const bool win = r * b.e < b.r * e;
  b.r = win ? r : b.r;
  b.e = win ? e : b.e;
  b.x = win ? x : b.x;
}

// Eight consecutive entries (group j of the chunk) of the correction race.
template <typename TT, typename TD, typename DK>
__device__ __forceinline__ void residual_group(const unsigned char* ts, const unsigned char* ds,
                                               int j, const ResidualTerms& rt, const DK& dk,
                                               int x0, Race& best) {
  float lt[8], ld[8], r[8];
  load8<TT>(ts, j, lt);
  load8<TD>(ds, j, ld);
  residual8(lt, ld, rt, r);
  const int xg = x0 + 8 * j;
  // both Philox words in straight-line code, so their round chains
  // interleave; candidates are selected without branches
  const uint4 w0 = vocab_words(dk, static_cast<uint32_t>(xg) >> 2);
  const uint4 w1 = vocab_words(dk, (static_cast<uint32_t>(xg) >> 2) + 1u);
  float e[8];
  neg_exp1_log2_x2(w0.x, w0.y, e[0], e[1]);
  neg_exp1_log2_x2(w0.z, w0.w, e[2], e[3]);
  neg_exp1_log2_x2(w1.x, w1.y, e[4], e[5]);
  neg_exp1_log2_x2(w1.z, w1.w, e[6], e[7]);
#pragma unroll
  for (int q = 0; q < 8; ++q) race_push(best, r[q], e[q], xg + q);
}

// Gumbel-max over the positive residual of one chunk.  Returns the warp's
// best (score lg2 r' - lg2 E + const, x); x = INT_MAX if the warp saw no
// positive residual.
template <typename TT, typename TD, bool kTma>
__device__ __forceinline__ void chunk_residual(const unsigned char* ts, const unsigned char* ds,
                                               const Hdr& h, const float4& st, const void* tgt,
                                               const void* drf, float c2, const Draw& d, int tid,
                                               float& bv, int& bi) {
  const ResidualTerms rt = residual_terms(c2, st);
  Race best{0.0f, -1.0f, INT_MAX};
  const int ng = kTma ? h.len / 8 : 0;
  const auto dk = chunk_draw(d);
  for (int j = tid; j < ng; j += kComputeThreads)
    residual_group<TT, TD>(ts, ds, j, rt, dk, h.x0, best);
  for (int e = 8 * ng + tid; e < h.len; e += kComputeThreads) {
    const int x = h.x0 + e;
    const float r = residual(load_elem<TT>(tgt, h.toff + e), load_elem<TD>(drf, h.doff + e), rt);
    race_push(best, r,
              neg_exp1_log2(word_of(vocab_words(d, static_cast<uint32_t>(x) >> 2), x & 3)), x);
  }
  bv = best.x == INT_MAX ? -INFINITY : lg2f(best.r) - lg2f(-best.e);
  bi = best.x;
  warp_argmax(bv, bi);
}

// Gumbel-max over l(x) / T of one chunk of the bonus row, in log2 units:
// the score is l(x) c2 + g(x) / ln 2 (c2 = log2(e) / T).
template <typename TT, bool kTma>
__device__ __forceinline__ void chunk_bonus(const unsigned char* ts, const Hdr& h,
                                            const void* tgt, float c2, const Draw& d, int tid,
                                            float& bv, int& bi) {
  bv = -INFINITY;
  bi = INT_MAX;
  const int ng = kTma ? h.len / 8 : 0;
  const auto dk = chunk_draw(d);
  for (int j = tid; j < ng; j += kComputeThreads) {
    float lt[8];
    load8<TT>(ts, j, lt);
    const int xg = h.x0 + 8 * j;
    const uint4 w0 = vocab_words(dk, static_cast<uint32_t>(xg) >> 2);
    const uint4 w1 = vocab_words(dk, (static_cast<uint32_t>(xg) >> 2) + 1u);
    float e[8];
    neg_exp1_log2_x2(w0.x, w0.y, e[0], e[1]);
    neg_exp1_log2_x2(w0.z, w0.w, e[2], e[3]);
    neg_exp1_log2_x2(w1.x, w1.y, e[4], e[5]);
    neg_exp1_log2_x2(w1.z, w1.w, e[6], e[7]);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float sc = fmaf(lt[q], c2, gumbel_log2(e[q]));
      const bool win = sc > bv;  // entries arrive in increasing x: first maximum kept
      bv = win ? sc : bv;
      bi = win ? xg + q : bi;
    }
  }
  for (int e = 8 * ng + tid; e < h.len; e += kComputeThreads) {
    const int x = h.x0 + e;
    const float sc =
        fmaf(load_elem<TT>(tgt, h.toff + e), c2,
             gumbel_log2(neg_exp1_log2(word_of(vocab_words(d, static_cast<uint32_t>(x) >> 2), x & 3))));
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

// Chunk statistics of a chunk retired unread (a NaN maximum, which no real
// chunk has): never zero, and it marks its row as not reduced in full.
constexpr unsigned long long kSkippedStats = 0x7fc00000ull;

// Rows decided / rejected, packed in the sequence state word.
__device__ __forceinline__ unsigned int decided_bits(unsigned long long st) {
  return static_cast<unsigned int>(st);
}
__device__ __forceinline__ unsigned int rejected_bits(unsigned long long st) {
  return static_cast<unsigned int>(st >> 32);
}
__device__ __forceinline__ unsigned int low_mask(int n) {  // bits 0..n-1, n <= 32
  return n >= 32 ? 0xffffffffu : (1u << n) - 1u;
}
// First rejection n (k when none is known), and whether every row 0..n is
// decided -- then n is the accepted length.
__device__ __forceinline__ bool resolved(unsigned long long st, int k, int& n) {
  const unsigned int rej = rejected_bits(st);
  n = rej ? __ffs(rej) - 1 : k;
  const unsigned int need = low_mask(n < k ? n + 1 : k);
  return (decided_bits(st) & need) == need;
}

// Place a chunk in the next stage of group g's ring (waits for the stage).
template <typename TT, typename TD, bool kTma>
__device__ __forceinline__ bool stoch_issue(const StochParams& p, Shared& sh,
                                            unsigned char* stages, int g, uint32_t& used,
                                            Hdr& h, const float4* stat) {
  h.x0 = h.c * p.ch;
  h.len = min(p.ch, p.V - h.x0);
  h.toff = static_cast<long long>(h.b) * p.t_sb + static_cast<long long>(h.i) * p.t_sp + h.x0;
  h.doff = static_cast<long long>(h.b) * p.d_sb + static_cast<long long>(h.i) * p.d_sp + h.x0;
  if (!SV_IN(p.ctrl, h.b, p.B) || !SV_IN(p.ctrl, h.i, p.k + 1) || !SV_IN(p.ctrl, h.c, p.nch) ||
      !SV_IN_RANGE(p.ctrl, h.toff, h.len, p.t_elems))
    h.toff = 0;  // (bounds-checked builds: a bad chunk reads the first row instead)
  if (h.kind != kKindBonus && !SV_IN_RANGE(p.ctrl, h.doff, h.len, p.d_elems)) h.doff = 0;
  const int s = group_stage(g, used);
  if (!mbar_wait(&sh.empty[s], group_phase(used) ^ 1u, p.ctrl)) return false;
  issue_chunk<TT, TD, kTma>(sh, stages + static_cast<size_t>(s) * kStageBytes, s, h, p.tgt,
                            p.drf, p.ch, h.kind != kKindBonus, stat);
  ++used;
  return true;
}

// A data-free item into group g's next stage: row (b, i) is complete (its
// last chunks were retired unread) and its epilogue merges it.
__device__ __forceinline__ bool stoch_push_row_done(Shared& sh, int g, uint32_t& used, int b,
                                                    int i, Ctrl* ctrl) {
  const int s = group_stage(g, used);
  if (!mbar_wait(&sh.empty[s], group_phase(used) ^ 1u, ctrl)) return false;
  sh.hdr[s].kind = kKindRowDone;
  sh.hdr[s].b = b;
  sh.hdr[s].i = i;
  mbar_arrive(&sh.full[s]);
  ++used;
  return true;
}

// Phase-2 chunk c of sequence b, whose accepted length n is known (the
// ready-list entry was acquired by the caller).  The correction's row
// statistics travel with the chunk as a 16-byte bulk copy.
template <typename TT, typename TD, bool kTma>
__device__ __forceinline__ bool stoch_issue_phase2(const StochParams& p, Shared& sh,
                                                   unsigned char* stages, int g,
                                                   uint32_t& used, int b, int n, int c,
                                                   int slot) {
  Hdr h;
  h.b = b;
  h.c = c;
  h.slot = slot;
  h.i = min(max(n, 0), p.k);  // clamped: no workspace content steers a read out of bounds
  const float4* stat = nullptr;
  if (h.i < p.k) {
    h.kind = kKindCorrection;
    stat = reinterpret_cast<const float4*>(&p.seq[b].mt);
    if (kTma) fence_proxy_async_global();
  } else {
    h.kind = kKindBonus;
  }
  return stoch_issue<TT, TD, kTma>(p, sh, stages, g, used, h, stat);
}

// Producer of compute group g: phase-1 chunks in position-major ticket order,
// then phase-2 chunks from the ready list.
//  - Phase 1 goes first: the decisions of the last positions, which only
//    phase-1 chunks advance, are the kernel's critical path, while the
//    phase-2 chunks of sequences resolved early can wait.  A producer that
//    served every ready phase-2 chunk before its drawn phase-1 tickets held
//    those tickets (and the rows they complete) for up to kDefer phase-2
//    computations.  Graph-timed, same box (us): B = 256, k = 8: 175.8 ->
//    168.4; B = 64, k = 4: 75.6 -> 73.9; B = 1: 22.6 -> 21.6 (SV_P1_FIRST 0
//    restores phase 2 first; SV_P2_RUN n > 0 lets n phase-2 chunks pass a
//    drawn phase-1 ticket, which measured no better than 0).
//  - Phase-1 tickets come two ahead of their use, and the state word of each
//    ticket's sequence is loaded one ticket ahead: a chunk of pair i whose
//    sequence already has a rejection before i is retired unread (its two
//    slots get kSkippedStats and it is counted on its row; if that completes
//    the row, a data-free item hands the row to the epilogue).  A retire
//    costs the producer about one L2 round trip (the state word it waits
//    for), and at the later positions nearly every ticket is retired; so
//    after a retired ticket the producer takes the next SV_BATCH (4)
//    consecutive tickets in one grab, and a ticket in the same row as the one
//    before it takes that ticket's state word (which only gains decisions)
//    instead of loading it again.  Batch 1 / 3 / 4 / 6 / 8, step of the four
//    bench calls (us): 244.5 / 236.1 / 234.4 / 237.6 / 240.3 (across two
//    runs; B = 256, k = 8: 170.2, 162.0, 162.9, 162.6, 163.7).
//  - Up to kDefer phase-2 tickets are held; their ready-list entries are
//    polled with relaxed loads (issued before the current chunk's stage wait,
//    read at the next iteration) and a chunk is issued once its entry is
//    visible.  When no phase-1 ticket is left, the producer waits (bounded)
//    for the oldest held entry.  Holding fewer tickets spreads a late
//    sequence's chunks over more producers.  kDefer 1 / 2 / 3, phase 1
//    first (us): B = 256: 162.5 / 163.8 / 164.7; B = 64: 70.0 / 70.8 / 72.0;
//    in another run 4 against 2: 168.0 against 163.9 and 73.7 against 71.1,
//    and 8 was slower still.
#ifndef SV_P2_RUN
#define SV_P2_RUN 0
#endif
#ifndef SV_P1_FIRST
#define SV_P1_FIRST 1
#endif
#ifndef SV_DEFER
#define SV_DEFER 1
#endif
#ifndef SV_HOLD
#define SV_HOLD 1
#endif
#ifndef SV_BATCH
#define SV_BATCH 4
#endif
template <typename TT, typename TD, bool kTma>
__device__ void stoch_producer(const StochParams& p, Shared& sh, unsigned char* stages, int g) {
  constexpr int kDefer = SV_DEFER;
  int run = 0;  // phase-2 chunks issued since the last phase-1 ticket was served
  constexpr unsigned int kNone = 0xffffffffu;
  Ctrl* ctrl = p.ctrl;
  const unsigned int nch = static_cast<unsigned int>(p.nch);
  const unsigned int B = static_cast<unsigned int>(p.B);
  uint32_t used = 0;  // uses of group g's stages issued
  bool ok = true;
  // the state word of the sequence of a phase-1 ticket past position 0
  auto state_of = [&](unsigned int t) -> unsigned long long {
    if (t >= p.total1) return 0ull;
    const unsigned int row = udiv(t, p.div_nch);
    const unsigned int i = udiv(row, p.div_B);
    return i > 0u ? ld_relaxed_u64(&p.seq[row - i * B].state) : 0ull;
  };
  // The first three phase-1 tickets of every producer are fixed by its index
  // (no atomic round trip before the first load); the counter hands out the
  // tickets after them.
  const unsigned int fixed = gridDim.x * kProducerWarps * 3u;
  const unsigned int first = (blockIdx.x * kProducerWarps + static_cast<unsigned int>(g)) * 3u;
  unsigned int t1 = first;
  unsigned int t1n = first + 1u;
  unsigned long long s1 = state_of(t1);
  unsigned long long s1n = state_of(t1n);
  // the tickets after t1n: a batch [bq_base, bq_base + bq_cnt) taken from
  // the counter in one grab, read one advance after its grab; after a
  // retired ticket the grab takes SV_BATCH tickets (consecutive chunks,
  // mostly of one row, whose state word is then read once), else one
  unsigned int bq_base = first + 2u, bq_pos = 0u, bq_cnt = 1u;
  bool last_retired = false;
  // Parked phase-1 tickets (p.park): a chunk of pair i >= 1 whose sequence
  // has rows before i undecided waits here, oldest first, while the producer
  // takes later tickets; it leaves once the state word decides it (a
  // rejection before i: retired unread; rows 0..i-1 all accepted: issued),
  // or, oldest first, when the queue is full or no new ticket is left.  A
  // parked chunk thus waits at least one stage wait, and its sequence's
  // state is read again just before it goes.  Queue of 1 / 2 / 3 / none
  // (graph-timed, same box, us): B = 256, k = 8: 167.7 / 170.4 / 173.8 /
  // 175.8; B = 64, k = 4: 61.1 / 63.2 / 65.8 / 68.9; B = 1: 22.0 / 24.1 /
  // 22.6 / 23.8; a queue of 8 was slower still (195.6 at B = 256).
  constexpr int kHold = SV_HOLD;
  unsigned int pt[kHold];
  unsigned long long ps[kHold];  // their sequences' state words as last polled
  int np = 0;
  auto pair_of = [&](unsigned int t) -> unsigned int {  // i of ticket t
    return udiv(udiv(t, p.div_nch), p.div_B);
  };
  auto parkable = [&](unsigned int t, unsigned long long st) -> bool {
    const unsigned int i = pair_of(t);
    const unsigned int need = low_mask(static_cast<int>(i));
    return i > 0u && (rejected_bits(st) & need) == 0u && (decided_bits(st) & need) != need;
  };
  // reload the parked tickets' state words (read at the next iteration)
  auto poll_parked = [&]() {
#pragma unroll
    for (int d = 0; d < kHold; ++d)
      if (d < np) {
        const unsigned int r = udiv(pt[d], p.div_nch);
        ps[d] = ld_relaxed_u64(&p.seq[r - udiv(r, p.div_B) * B].state);
      }
  };
  unsigned int dt[kDefer];         // held phase-2 tickets, oldest first
  unsigned long long dv[kDefer];   // their ready-list entries as last polled
  int nd = 0;
  unsigned int t2p = kNone;        // a phase-2 grab in flight
  bool t2_done = p.total2 == 0u;
  // Retired chunks whose count is checked later (the counter's old value
  // arrives while the producer goes on): a count that completes the row
  // hands the row to the epilogue.  No resolution waits on a retired row (it
  // lies past a rejection), so the hand-over may lag.
  // One entry: a retire's count is checked at the next iteration, so a row
  // that its retires complete reaches the epilogue soonest.  Queue of 1 / 2
  // / 3 / 4 / 8, step of the four bench calls (us, two runs): 228.3 / 230.1
  // / 234.7 / 234.1 / 252.9; B = 256, k = 8: 157.3 / 159.8 / 161.6 / 162.5 /
  // 175.1.
#ifndef SV_SKQ
#define SV_SKQ 1
#endif
  constexpr int kSk = SV_SKQ;
  int skb[kSk], ski[kSk];
  unsigned int sko[kSk];
  int nsk = 0;
  auto settle_retired = [&]() -> bool {
#pragma unroll
    for (int d = 0; d < kSk; ++d)
      if (d < nsk && sko[d] == nch - 1u && !stoch_push_row_done(sh, g, used, skb[d], ski[d], ctrl))
        return false;
    nsk = 0;
    return true;
  };
  while (ok) {
    // (the held arrays are indexed with constants only, so they stay in
    // registers and a poll's load is not waited for until it is read)
    if (t2p != kNone) {  // the phase-2 grab of the previous iteration joins the queue
      if (t2p < p.total2) {
        const unsigned long long v0 =
            p.k == 0 ? (static_cast<unsigned long long>(udiv(t2p, p.div_nch)) + 1ull) : 0ull;
#pragma unroll
        for (int d = 0; d < kDefer; ++d)
          if (d == nd) {
            dt[d] = t2p;
            dv[d] = v0;
          }
        ++nd;
      } else {
        t2_done = true;
      }
      t2p = kNone;
    }
    // a held phase-2 chunk whose sequence is ready goes first
    int rd = -1;
#pragma unroll
    for (int d = kDefer - 1; d >= 0; --d)
      if (d < nd && dv[d] != 0ull) rd = d;
    if (rd < 0 && t1 >= p.total1 && np == 0 && nd > 0) {
      if (!settle_retired()) {
        ok = false;
        break;
      }
      // nothing else to do: wait (bounded) for the oldest held entry
      const unsigned long long* e = p.list + udiv(dt[0], p.div_nch);
      unsigned long long v = ld_relaxed_u64(e);
      const unsigned long long w0 = global_ns();
      for (unsigned int spin = 1; v == 0ull; ++spin) {
        __nanosleep(64);
        v = ld_relaxed_u64(e);
        if ((spin & 63u) == 0u) {
          if (aborted(ctrl)) break;
          if (global_ns() - w0 > kWaitLimitNs) {
            atomicOr(&ctrl->flags, kFlagTimeout);
            break;
          }
        }
      }
      if (v == 0ull) {
        ok = false;
        break;
      }
      dv[0] = v;
      rd = 0;
    }
    // keep up to kDefer phase-2 tickets in hand (the atomic's result is used
    // at the next iteration)
    if (!t2_done && nd < kDefer) t2p = atomicAdd(&ctrl->ticket2, 1u);
    if (rd >= 0 && (t1 < p.total1 || np > 0) &&
        (SV_P1_FIRST || (SV_P2_RUN > 0 && run >= SV_P2_RUN)))
      rd = -1;  // the drawn phase-1 ticket goes first; the ready entry stays held
    if (rd >= 0) {
      ++run;
      unsigned long long v = 0ull;
      unsigned int tsel = 0u;
#pragma unroll
      for (int d = 0; d < kDefer; ++d)
        if (d == rd) {
          v = dv[d];
          tsel = dt[d];
        }
      const unsigned int slot = udiv(tsel, p.div_nch);
      const unsigned int c = tsel - slot * nch;
      if (!SV_IN(ctrl, slot, p.B)) continue;
#pragma unroll
      for (int d = 0; d < kDefer - 1; ++d)
        if (d >= rd && d + 1 < nd) {
          dt[d] = dt[d + 1];
          dv[d] = dv[d + 1];
        }
      --nd;
      // poll the rest now; the stage wait below overlaps the round trip
#pragma unroll
      for (int d = 0; d < kDefer; ++d)
        if (d < nd && dv[d] == 0ull) dv[d] = ld_relaxed_u64(p.list + udiv(dt[d], p.div_nch));
      if (p.k > 0) fence_acq_rel_gpu();  // acquire: the resolver's record is visible
      // (clamped so that no workspace content can steer a read outside the
      // tensors)
      const int b = static_cast<int>(min(static_cast<unsigned int>(v) - 1u, B - 1u));
      const int n = static_cast<int>(v >> 32);
      ok = stoch_issue_phase2<TT, TD, kTma>(p, sh, stages, g, used, b, n, static_cast<int>(c),
                                            static_cast<int>(slot));
      if (ok) ok = settle_retired();  // their counts arrived during the stage wait
      continue;
    }
#pragma unroll
    for (int d = 0; d < kDefer; ++d)
      if (d < nd && dv[d] == 0ull) dv[d] = ld_relaxed_u64(p.list + udiv(dt[d], p.div_nch));
    if (t1 < p.total1 || np > 0) {
      // a parked ticket that its state decides (oldest first); else, with
      // the queue full or no new ticket left, the oldest; else a new ticket,
      // parked if it can be
      int pr = -1;
#pragma unroll
      for (int d = kHold - 1; d >= 0; --d)
        if (d < np && !parkable(pt[d], ps[d])) pr = d;
      if (pr < 0 && np > 0 && (t1 >= p.total1 || (np == kHold && parkable(t1, s1)))) pr = 0;
      unsigned int tk;
      unsigned long long sk;
      if (pr >= 0) {
        tk = 0u;
        sk = 0ull;
#pragma unroll
        for (int d = 0; d < kHold; ++d)
          if (d == pr) {
            tk = pt[d];
            sk = ps[d];
          }
#pragma unroll
        for (int d = 0; d < kHold - 1; ++d)
          if (d >= pr && d + 1 < np) {
            pt[d] = pt[d + 1];
            ps[d] = ps[d + 1];
          }
        --np;
      } else {
        tk = t1;
        sk = s1;
        // advance the ticket pipeline before this chunk's stage wait; the
        // state of a ticket in the same row as the one before it is that
        // ticket's (a state word only gains decisions)
        t1 = t1n;
        s1 = s1n;
        t1n = bq_base + bq_pos;
        ++bq_pos;
        s1n = (t1n < p.total1 && t1 < p.total1 && udiv(t1n, p.div_nch) == udiv(t1, p.div_nch))
                  ? s1
                  : state_of(t1n);
        if (bq_pos == bq_cnt) {  // the batch is used up: grab the next one now
          bq_cnt = (SV_BATCH > 1 && last_retired) ? SV_BATCH : 1u;
          bq_base = fixed + atomicAdd(&ctrl->ticket, bq_cnt);
          bq_pos = 0u;
        }
        if (p.park && np < kHold && parkable(tk, sk)) {
#pragma unroll
          for (int d = 0; d < kHold; ++d)
            if (d == np) {
              pt[d] = tk;
              ps[d] = sk;
            }
          ++np;
          poll_parked();
          continue;
        }
      }
      poll_parked();  // the stage wait below overlaps the round trips
      const unsigned int row = udiv(tk, p.div_nch);
      const unsigned int i = udiv(row, p.div_B);
      Hdr h;
      h.kind = kKindStats;
      h.b = static_cast<int>(row - i * B);
      h.i = static_cast<int>(i);
      h.c = static_cast<int>(tk - row * nch);
      const unsigned int rej = rejected_bits(sk);
      run = 0;
      if (rej & low_mask(h.i)) {  // a pair before this one was rejected: retire unread
        if (!SV_IN(ctrl, h.b, p.B) || !SV_IN(ctrl, h.i, p.k) || !SV_IN(ctrl, h.c, p.nch)) continue;
        unsigned long long* slot =
            p.p1 + ((static_cast<size_t>(h.b) * p.k + h.i) * nch + h.c) * 2;
        st_relaxed_u64(slot, kSkippedStats);
        st_relaxed_u64(slot + 1, kSkippedStats);
        if (nsk == kSk && !settle_retired()) {
          ok = false;
          break;
        }
        const unsigned int old = atomicAdd(&p.rc[static_cast<size_t>(h.b) * p.k + h.i], 1u);
#pragma unroll
        for (int d = 0; d < kSk; ++d)
          if (d == nsk) {
            skb[d] = h.b;
            ski[d] = h.i;
            sko[d] = old;
          }
        ++nsk;
        last_retired = true;
        continue;
      }
      last_retired = false;
      ok = stoch_issue<TT, TD, kTma>(p, sh, stages, g, used, h, nullptr);
      if (ok) ok = settle_retired();  // their counts arrived during the stage wait
      continue;
    }
    if (nd == 0 && t2_done && t2p == kNone) {  // no work left
      ok = settle_retired();
      break;
    }
    if (nd == 0 && t2p != kNone) continue;           // a grab in flight
  }
  if (ok) {
    push_group_end(sh, g, used, ctrl);
    // the last producer to leave rewinds every counter
    if (atomicAdd(&ctrl->exits, 1u) == gridDim.x * kProducerWarps - 1) {
      atomicExch(&ctrl->ticket, 0u);
      atomicExch(&ctrl->ticket2, 0u);
      atomicExch(&ctrl->resolved, 0u);
      atomicExch(&ctrl->exits, 0u);
    }
  } else if (kTma) {
    drain_group_stages(sh, g, used);
  }
}

template <typename TT, typename TD, bool kTma>
__device__ void stoch_compute(const StochParams& p, Shared& sh, unsigned char* stages, int w,
                              int lane) {
  const int group = w / kGroupWarps;
  w %= kGroupWarps;
  const int tid = w * 32 + lane;
  for (uint32_t use = group;; use += kComputeGroups) {
    const int s = use % kStages;
    if (!mbar_wait(&sh.full[s], (use / kStages) & 1u, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd || h.kind == kKindRowDone) {
      if (lane == 0) mbar_arrive(&sh.rfull[s]);
      if (h.kind == kKindEnd) break;
      continue;
    }
    const unsigned char* ts = stages + static_cast<size_t>(s) * kStageBytes;
    const unsigned char* ds = ts + static_cast<size_t>(p.ch) * Elem<TT>::kBytes;
    float4 r;
    if (h.kind == kKindStats) {
      if (kTma) {
        r = chunk_stats_pair<TT, TD>(ts, ds, h, p.tgt, p.drf, p.c2, tid);
      } else {
        float m1, s1, m2, s2;
        chunk_stats<TT>(ts, h.nvec_t, p.tgt, h.toff, h.len, p.c2, tid, m1, s1);
        chunk_stats<TD>(ds, h.nvec_d, p.drf, h.doff, h.len, p.c2, tid, m2, s2);
        r = make_float4(m1, s1, m2, s2);
      }
    } else {
      const Draw d{p.key0, p.key1, static_cast<uint32_t>(h.i),
                   static_cast<uint32_t>(h.b) + p.seq_offset,
                   h.kind == kKindCorrection ? kTagCorrection : kTagBonus};
      float bv;
      int bi;
      if (h.kind == kKindCorrection)
        chunk_residual<TT, TD, kTma>(ts, ds, h, sh.rstat[s], p.tgt, p.drf, p.c2, d, tid, bv,
                                     bi);
      else
        chunk_bonus<TT, kTma>(ts, h, p.tgt, p.c2, d, tid, bv, bi);
      r = make_float4(bv, __int_as_float(bi), 0.0f, 0.0f);
    }
    if (lane == 0) {
      sh.res[s][w] = r;
      mbar_arrive(&sh.rfull[s]);
    }
  }
}

// Read a published partial: the load is issued at once; only a slot whose
// store is not visible yet is polled.
__device__ __forceinline__ unsigned long long take(unsigned long long* slot, unsigned long long v,
                                                   Ctrl* ctrl) {
  if (v == 0ull) v = poll_u64(slot, ctrl);
  *slot = 0ull;
  return v;
}

// Resolution of sequence b (one warp), once its accepted length n is known:
// the committed drafts and the -1 padding, the row-n statistics for the
// phase-2 draw (consumed from the rejected row's record; `own`, when not null,
// holds them already -- the caller merged row n -- and the record is only
// cleared), and an entry in the ready list that releases its phase-2 chunks.
__device__ void resolve_sequence(const StochParams& p, int b, int n, int lane,
                                 const float4* own) {
  const int k = p.k;
  if (!SV_IN(p.ctrl, b, p.B) || !SV_IN(p.ctrl, n, k + 1)) return;
  float4 st = make_float4(0.0f, 1.0f, 0.0f, 1.0f);
  if (n < k) {
    unsigned long long* row = p.r1 + (static_cast<size_t>(b) * k + n) * 2;
    if (own) {
      st = *own;
      if (lane == 0) {  // the lane that wrote the record
        row[0] = 0ull;
        row[1] = 0ull;
      }
    } else {
      float m, sm;
      unpack_stats(take(row, ld_relaxed_u64(row), p.ctrl), m, sm);
      st.x = m;
      st.y = sm;
      unpack_stats(take(row + 1, ld_relaxed_u64(row + 1), p.ctrl), m, sm);
      st.z = m;
      st.w = sm;
    }
  }
  int* out = p.out_tokens + static_cast<size_t>(b) * (k + 1);
  for (int i = lane; i <= k; i += 32)
    if (i != n) out[i] = i < n ? __ldg(p.tokens + static_cast<size_t>(b) * k + i) : -1;
  if (lane == 0) {
    p.accepted_len[b] = n;
    SeqRec* r = p.seq + b;
    r->n = n;
    r->mt = st.x;
    r->ist = 1.0f / st.y;
    r->md = st.z;
    r->isd = 1.0f / st.w;
    const unsigned int slot = atomicAdd(&p.ctrl->resolved, 1u);
    // the release store below orders the record before the entry; the
    // statistics are bulk-copied by the producer (async proxy)
    fence_proxy_async_global();
    if (slot < static_cast<unsigned int>(p.B))  // (each sequence resolves once: always true)
      st_release_u64(p.list + slot, (static_cast<unsigned long long>(n) << 32) |
                                        (static_cast<unsigned int>(b) + 1u));
  }
}

// Row merge of pair i of sequence b (one warp, one lane per chunk): the row
// statistics, then the row's own acceptance decision -- p_i(x_i), q_i(x_i),
// u_i, accept while u_i q < p -- published in the sequence state word with one
// atomicOr.  The merge whose update makes rows 0..n decided (n the first
// rejection, or k) resolves the sequence; the merge that decides the last row
// clears what the resolution left (statistics of later rejected rows) and the
// state word.  A row with a chunk retired unread lies past a known rejection:
// it is marked decided without a decision.
template <typename TT, typename TD>
__device__ void merge_row(const StochParams& p, int b, int i, int lane) {
  const int k = p.k;
  if (!SV_IN(p.ctrl, b, p.B) || !SV_IN(p.ctrl, i, k)) return;
  unsigned long long* slot = p.p1 + (static_cast<size_t>(b) * k + i) * p.nch * 2;
  float MT = -INFINITY, ST = 0.0f, MD = -INFINITY, SD = 0.0f;
  bool skipped = false;
  for (int c = lane; c < p.nch; c += 32) {
    const unsigned long long vt0 = ld_relaxed_u64(slot + 2 * c);
    const unsigned long long vd0 = ld_relaxed_u64(slot + 2 * c + 1);
    const unsigned long long vt = take(slot + 2 * c, vt0, p.ctrl);
    const unsigned long long vd = take(slot + 2 * c + 1, vd0, p.ctrl);
    if (vt == kSkippedStats) {
      skipped = true;
      continue;
    }
    float m, s;
    unpack_stats(vt, m, s);
    merge_stats(MT, ST, m, s);
    unpack_stats(vd, m, s);
    merge_stats(MD, SD, m, s);
  }
  skipped = __any_sync(0xffffffffu, skipped);
  const float4 w = warp_stats2(make_float4(MT, ST, MD, SD));
  bool rejected = false;
  if (lane == 0) {
    const int x = __ldg(p.tokens + static_cast<size_t>(b) * k + i);
    const bool valid = x >= 0 && x < p.V;
    if (!valid) atomicOr(&p.ctrl->flags, kFlagInvalidToken);
    float pt = -1.0f, qd = -1.0f;  // -1: not read in full (past a rejection)
    if (!skipped) {
      pt = 0.0f;
      qd = 0.0f;
      const long long ot =
          static_cast<long long>(b) * p.t_sb + static_cast<long long>(i) * p.t_sp + x;
      const long long od =
          static_cast<long long>(b) * p.d_sb + static_cast<long long>(i) * p.d_sp + x;
      if (valid && SV_IN(p.ctrl, ot, p.t_elems) && SV_IN(p.ctrl, od, p.d_elems)) {
        const float lt = load_elem<TT>(p.tgt, ot);
        const float ld = load_elem<TD>(p.drf, od);
        pt = ex2f(fmaf(lt, p.c2, -w.x)) / w.y;
        qd = ex2f(fmaf(ld, p.c2, -w.z)) / w.w;
      }
      const uint4 u = philox10(
          make_uint4(0u, static_cast<uint32_t>(i), static_cast<uint32_t>(b) + p.seq_offset,
                     kTagAccept),
          p.key0, p.key1);
      rejected = !(valid && (accept_uniform(u.x) * qd < pt));
      if (rejected) {  // the statistics a resolution at this row reads
        unsigned long long* row = p.r1 + (static_cast<size_t>(b) * k + i) * 2;
        st_relaxed_u64(row, pack_stats(w.x, w.y));
        st_relaxed_u64(row + 1, pack_stats(w.z, w.w));
      }
    }
    if (p.probs) {
      float* pr = p.probs + (static_cast<size_t>(b) * k + i) * 2;
      pr[0] = pt;
      pr[1] = qd;
    }
  }
  unsigned long long old = 0ull, bits = 0ull;
  if (lane == 0) {
    p.rc[static_cast<size_t>(b) * k + i] = 0u;
    bits = (1ull << i) | (rejected ? (1ull << (32 + i)) : 0ull);
    // release: this row's record before the state update; acquire: the
    // records of the rows whose bits it returns
    old = atom_or_acq_rel_u64(&p.seq[b].state, bits);
  }
  old = __shfl_sync(0xffffffffu, old, 0);
  bits = __shfl_sync(0xffffffffu, bits, 0);
  rejected = __shfl_sync(0xffffffffu, rejected ? 1 : 0, 0) != 0;
  const unsigned long long now = old | bits;
  int n_old, n_now;
  const bool was = resolved(old, k, n_old);
  if (!was && resolved(now, k, n_now))
    resolve_sequence(p, b, n_now, lane, rejected && n_now == i ? &w : nullptr);
  if (decided_bits(old) != low_mask(k) && decided_bits(now) == low_mask(k)) {
    // the last row of the sequence: clear the records of rejected rows past
    // n (rows retired unread are never marked rejected and wrote none)
    resolved(now, k, n_now);
    const unsigned int later = rejected_bits(now) & ~low_mask(n_now + 1) & low_mask(k);
    for (unsigned int m = later; m;) {
      const int j = __ffs(m) - 1;
      m &= m - 1u;
      unsigned long long* row = p.r1 + (static_cast<size_t>(b) * k + j) * 2;
      if (lane < 2) take(row + lane, ld_relaxed_u64(row + lane), p.ctrl);
    }
    if (lane == 0) p.seq[b].state = 0ull;
  }
}

// Phase-2 finalize of sequence b (one warp): the largest chunk key gives the
// token at position n.  With no positive residual mass the token is drawn
// from p_n with the same CORRECTION stream (slow path, one warp).  Clears the
// sequence's record and its ready-list entry.
template <typename TT>
__device__ void finalize_sample(const StochParams& p, int b, int n, int entry, int lane) {
  const int k = p.k;
  if (!SV_IN(p.ctrl, b, p.B) || !SV_IN(p.ctrl, n, k + 1) || !SV_IN(p.ctrl, entry, p.B)) return;
  unsigned long long key = 0ull;
  unsigned long long* slot = p.p2 + static_cast<size_t>(b) * p.nch;
  for (int c = lane; c < p.nch; c += 32) {
    const unsigned long long v = take(slot + c, ld_relaxed_u64(slot + c), p.ctrl);
    key = v > key ? v : key;
  }
  key = warp_max_u64(key);
  int tok;
  if (key <= kNoCandidate) {
    if (lane == 0) atomicOr(&p.ctrl->flags, kFlagResidualFallback);
    const Draw d{p.key0, p.key1, static_cast<uint32_t>(n),
                 static_cast<uint32_t>(b) + p.seq_offset, kTagCorrection};
    const long long off = static_cast<long long>(b) * p.t_sb + static_cast<long long>(n) * p.t_sp;
    float bv = -INFINITY;
    int bi = INT_MAX;
    const int V = SV_IN_RANGE(p.ctrl, off, p.V, p.t_elems) ? p.V : 0;
    for (int x = lane; x < V; x += 32) {
      const float sc = fmaf(load_elem<TT>(p.tgt, off + x), p.c2,
                            gumbel_log2(neg_exp1_log2(
                                word_of(vocab_words(d, static_cast<uint32_t>(x) >> 2), x & 3))));
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
    if (k > 0) p.list[entry] = 0ull;
    r->n = 0;
    r->mt = r->ist = r->md = r->isd = 0.0f;
    r->cnt2 = 0u;
  }
}

// An arrival whose counter value is checked later.
struct Pending {
  int kind;           // 0: none, kKindStats (row counter) or kKindCorrection (cnt2)
  int b, i;           // sequence; position (phase-1 row, or phase-2 row n)
  int slot;           // phase 2: the sequence's ready-list entry
  unsigned int old;   // counter value before this arrival (lane 0)
};

template <typename TT, typename TD>
__device__ __forceinline__ void resolve(const StochParams& p, Pending& pd, int lane) {
  if (pd.kind == 0) return;
  const unsigned int last = static_cast<unsigned int>(p.nch) - 1u;
  if (__shfl_sync(0xffffffffu, pd.old == last ? 1 : 0, 0)) {
    if (pd.kind == kKindStats)
      merge_row<TT, TD>(p, pd.b, pd.i, lane);
    else
      finalize_sample<TT>(p, pd.b, pd.i, pd.slot, lane);
  }
  pd.kind = 0;
}

template <typename TT, typename TD>
__device__ void stoch_epilogue(const StochParams& p, Shared& sh, int group, int lane) {
  Pending pd{0, 0, 0, 0, 0u};
  for (uint32_t use = group;; use += kComputeGroups) {
    const int s = use % kStages;
    const uint32_t parity = (use / kStages) & 1u;
    // nothing to overlap with: settle the previous arrival before blocking
    if (pd.kind != 0 && !mbar_try_wait(&sh.rfull[s], parity)) resolve<TT, TD>(p, pd, lane);
    if (!mbar_wait(&sh.rfull[s], parity, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd) break;
    if (h.kind == kKindRowDone) {  // every chunk of the row is counted: merge it
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.empty[s]);
      resolve<TT, TD>(p, pd, lane);
      merge_row<TT, TD>(p, h.b, h.i, lane);
      continue;
    }
    float4 r = lane < kGroupWarps ? sh.res[s][lane]
                                  : make_float4(-INFINITY, __int_as_float(INT_MAX), 0.f, 0.f);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.empty[s]);
    if (!SV_IN(p.ctrl, h.b, p.B) || !SV_IN(p.ctrl, h.c, p.nch) ||
        !SV_IN(p.ctrl, h.i, h.kind == kKindStats ? p.k : p.k + 1))
      continue;
    unsigned int old = 0u;
    Pending next;
    if (h.kind == kKindStats) {
      if (lane >= kGroupWarps) r = make_float4(-INFINITY, 0.0f, -INFINITY, 0.0f);
      r = warp_stats2(r);
      if (lane == 0) {
        unsigned long long* slot =
            p.p1 + ((static_cast<size_t>(h.b) * p.k + h.i) * p.nch + h.c) * 2;
        st_relaxed_u64(slot, pack_stats(r.x, r.y));
        st_relaxed_u64(slot + 1, pack_stats(r.z, r.w));
        old = atomicAdd(&p.rc[static_cast<size_t>(h.b) * p.k + h.i], 1u);
      }
      next = Pending{kKindStats, h.b, h.i, 0, old};
    } else {
      float v = r.x;
      int i = __float_as_int(r.y);
      warp_argmax(v, i);
      if (lane == 0) {
        st_relaxed_u64(p.p2 + static_cast<size_t>(h.b) * p.nch + h.c,
                       i == INT_MAX ? kNoCandidate : make_key(v, i));
        old = atomicAdd(&p.seq[h.b].cnt2, 1u);
      }
      next = Pending{kKindCorrection, h.b, h.i, h.slot, old};
    }
    resolve<TT, TD>(p, pd, lane);
    pd = next;
  }
  resolve<TT, TD>(p, pd, lane);
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
      mbar_init(&sh.rfull[s], kGroupWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();
  dep_enter();
  if (warp < kProducerWarps) {
    if (lane == 0) stoch_producer<TT, TD, kTma>(p, sh, stages, warp);
  } else if (warp < kProducerWarps + kComputeWarps) {
    stoch_compute<TT, TD, kTma>(p, sh, stages, warp - kProducerWarps, lane);
  } else {
    stoch_epilogue<TT, TD>(p, sh, warp - kProducerWarps - kComputeWarps, lane);
  }
}

// ================================================================ argmax

// Hand row (b, r), whose last chunk this producer just retired unread, to
// the epilogue of the group that takes the next stage: a data-free item.
__device__ __forceinline__ bool push_row_done(Shared& sh, uint32_t& use, int b, int r,
                                              Ctrl* ctrl, int g) {
  const int s = g < 0 ? static_cast<int>(use % kStages) : group_stage(g, use);
  const uint32_t ph = g < 0 ? (use / kStages) & 1u : group_phase(use);
  if (!mbar_wait(&sh.empty[s], ph ^ 1u, ctrl)) return false;
  sh.hdr[s].kind = kKindRowDone;
  sh.hdr[s].b = b;
  sh.hdr[s].i = r;
  mbar_arrive(&sh.full[s]);
  ++use;
  return true;
}

// kRowStride: rows or tree form, row h.i of the sequence at stride sg.
// kEarly (plain mode): tickets are position-major, and a chunk of a row past
// its branch's first known mismatch is retired without being read: its slot
// gets kSkippedKey and it is counted on the row like a reduced chunk.  Rows up
// to the branch's first mismatch are never retired (a mismatch is only known
// once its row has been reduced in full), so the row argmaxes the finalize
// uses are exact.
// g < 0: the one producer of the CTA, alternating the groups' stages; g >= 0:
// the producer of compute group g, filling that group's stages only.
template <typename TT, bool kTma, bool kRowStride, bool kEarly>
__device__ void argmax_producer(const ArgmaxParams& p, Shared& sh, unsigned char* stages, int g) {
  Ctrl* ctrl = p.ctrl;
  const unsigned int per_seq = static_cast<unsigned int>(p.R) * static_cast<unsigned int>(p.nch);
  const unsigned int nch = static_cast<unsigned int>(p.nch);
  const unsigned int BG = static_cast<unsigned int>(p.B) * static_cast<unsigned int>(p.G);
  uint32_t use = 0;
  bool ok = true;
  // plain mode: the branch state of a position >= 1 ticket, loaded one
  // ticket ahead so that its round trip overlaps the current ticket's work
  auto branch_state = [&](unsigned int t) -> unsigned int {
    if (!kEarly || t >= p.total) return 0u;
    const unsigned int row = udiv(t, p.div_nch);
    const unsigned int pos = udiv(row, p.div_bg);
    return pos > 0u && SV_IN(ctrl, row - pos * BG, BG) ? ld_relaxed_u32(p.dead + (row - pos * BG))
                                                        : 0u;
  };
  // The first grab of every CTA is fixed by its index (no atomic round trip
  // before the first load); the counter hands out the tickets after them.
  const unsigned int fixed = gridDim.x * kArgmaxProducers * kGrabArgmax;
  unsigned int base = (blockIdx.x * kArgmaxProducers + static_cast<unsigned int>(g < 0 ? 0 : g)) *
                      kGrabArgmax;
  unsigned int dv_next = branch_state(base);
  while (ok && base < p.total) {
    const unsigned int next = fixed + atomicAdd(&ctrl->ticket, kGrabArgmax);
    // retired chunks of the current row, counted with one atomic per run
    int sk_b = -1, sk_r = 0;
    unsigned int sk_n = 0u;
#pragma unroll 1
    for (unsigned int j = 0; j < kGrabArgmax; ++j) {
      const unsigned int t = base + j;
      if (t >= p.total) break;
      const unsigned int dv = dv_next;
      dv_next = branch_state(j + 1 < kGrabArgmax ? t + 1 : next);
      Hdr h;
      h.kind = kKindArgmax;
      int pos = 0;
      if (kEarly) {
        const unsigned int row = udiv(t, p.div_nch);
        const unsigned int ps = udiv(row, p.div_bg);
        const unsigned int bg = row - ps * BG;
        const unsigned int b = udiv(bg, p.div_g);
        const unsigned int g = bg - b * static_cast<unsigned int>(p.G);
        pos = static_cast<int>(ps);
        h.b = static_cast<int>(b);
        h.i = static_cast<int>(g) * (p.k + 1) + pos;
        h.c = static_cast<int>(t - row * nch);
      } else {
        const unsigned int b = udiv(t, p.div_seq);
        const unsigned int rem = t - b * per_seq;
        const unsigned int i = udiv(rem, p.div_nch);
        h.b = static_cast<int>(b);
        h.i = static_cast<int>(i);
        h.c = static_cast<int>(rem - i * nch);
      }
      if (kEarly && sk_b >= 0 && (h.b != sk_b || h.i != sk_r)) {  // a run of retired chunks ends
        const unsigned int old = atomicAdd(&p.rc[static_cast<size_t>(sk_b) * p.R + sk_r], sk_n);
        if (old + sk_n == nch) ok = push_row_done(sh, use, sk_b, sk_r, ctrl, g);
        sk_b = -1;
        sk_n = 0u;
        if (!ok) break;
      }
      if (!SV_IN(ctrl, h.b, p.B) || !SV_IN(ctrl, h.i, p.R) || !SV_IN(ctrl, h.c, p.nch)) continue;
      if (kEarly && dv != 0u && 64 - static_cast<int>(dv) < pos) {
        st_relaxed_u64(p.slots + (static_cast<size_t>(h.b) * p.R + h.i) * nch + h.c, kSkippedKey);
        sk_b = h.b;
        sk_r = h.i;
        ++sk_n;
        continue;
      }
      h.x0 = h.c * p.ch;
      h.len = min(p.ch, p.V - h.x0);
      if (kRowStride) {
        h.toff = static_cast<long long>(h.b) * p.sb + static_cast<long long>(h.i) * p.sg + h.x0;
      } else {
        const int g = h.i / (p.k + 1), ps = h.i - g * (p.k + 1);
        h.toff = static_cast<long long>(h.b) * p.sb + static_cast<long long>(g) * p.sg +
                 static_cast<long long>(ps) * p.sp + h.x0;
      }
      h.doff = 0;
      if (!SV_IN_RANGE(ctrl, h.toff, h.len, p.t_elems)) h.toff = 0;
      const int s = g < 0 ? static_cast<int>(use % kStages) : group_stage(g, use);
      const uint32_t ph = g < 0 ? (use / kStages) & 1u : group_phase(use);
      if (!mbar_wait(&sh.empty[s], ph ^ 1u, ctrl)) {
        ok = false;
        break;
      }
      issue_chunk<TT, TT, kTma>(sh, stages + static_cast<size_t>(s) * kStageBytes, s, h, p.tgt,
                                nullptr, p.ch, false, nullptr);
      ++use;
    }
    if (kEarly && ok && sk_b >= 0) {
      const unsigned int old = atomicAdd(&p.rc[static_cast<size_t>(sk_b) * p.R + sk_r], sk_n);
      if (old + sk_n == nch) ok = push_row_done(sh, use, sk_b, sk_r, ctrl, g);
    }
    base = next;
  }
  if (ok) {
    if (g < 0)
      push_end(sh, use, ctrl);
    else
      push_group_end(sh, g, use, ctrl);
    leave_grid(ctrl, static_cast<unsigned int>(kArgmaxProducers));
  } else if (kTma) {
    if (g < 0)
      drain_stages(sh, use);
    else
      drain_group_stages(sh, g, use);
  }
}

// Argmax kernel modes, one instantiation each so that every kernel carries
// only its own finalize: plain (greedy and multi-candidate), rows form, tree,
// threshold acceptance (row softmax statistics as well).
enum : int { kArgPlain = 0, kArgRows = 1, kArgTree = 2, kArgThreshold = 3 };

template <typename TT, bool kTma, int kMode>
__device__ void argmax_compute(const ArgmaxParams& p, Shared& sh, unsigned char* stages, int w,
                               int lane) {
  const int group = w / kGroupWarps;
  w %= kGroupWarps;
  const int tid = w * 32 + lane;
  for (uint32_t use = group;; use += kComputeGroups) {
    const int s = use % kStages;
    if (!mbar_wait(&sh.full[s], (use / kStages) & 1u, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd || h.kind == kKindRowDone) {
      if (lane == 0) mbar_arrive(&sh.rfull[s]);
      if (h.kind == kKindEnd) break;
      continue;
    }
    float bv;
    int bi;
    float4 r = make_float4(0.0f, 0.0f, -INFINITY, 0.0f);
    if (kMode == kArgThreshold && h.i < p.k) {  // row statistics too
      if (kTma) {
        r = chunk_argmax_stats_regs<TT>(stages + static_cast<size_t>(s) * kStageBytes, h, p.tgt,
                                        p.c2, tid, sh, s, lane);
      } else {
        chunk_argmax<TT>(stages + static_cast<size_t>(s) * kStageBytes, h, p.tgt, tid, bv, bi);
        float m, sm;
        chunk_stats<TT>(stages + static_cast<size_t>(s) * kStageBytes, h.nvec_t, p.tgt, h.toff,
                        h.len, p.c2, tid, m, sm);
        r = make_float4(bv, __int_as_float(bi), m, sm);
      }
    } else {
      if (kTma)
        chunk_argmax_regs<TT>(stages + static_cast<size_t>(s) * kStageBytes, h, p.tgt, tid, bv,
                              bi);
      else
        chunk_argmax<TT>(stages + static_cast<size_t>(s) * kStageBytes, h, p.tgt, tid, bv, bi);
      r.x = bv;
      r.y = __int_as_float(bi);
    }
    if (lane == 0) {
      sh.res[s][w] = r;
      mbar_arrive(&sh.rfull[s]);
    }
  }
}

// Threshold acceptance, finalize of sequence b (one warp, lane i = position
// i): log2 p_i(x_i) = l_i(x_i) c2 - m_i - lg2 s_i from the row statistics; an
// inclusive prefix sum gives the log2 score of each prefix; n = the first
// position whose prefix falls below the threshold (or k); the extra token
// is row n's argmax.
__device__ void finalize_threshold(const ArgmaxParams& p, int b, int lane) {
  const int k = p.k, R = p.R, V = p.V;
  unsigned long long* keys = p.rkey + static_cast<size_t>(b) * R;
  unsigned long long* stats = p.rstats + static_cast<size_t>(b) * R;
  const unsigned long long kv = lane <= k ? take(keys + lane, ld_relaxed_u64(keys + lane), p.ctrl)
                                          : 0ull;
  const unsigned long long k32 =
      (k == 32 && lane == 0) ? take(keys + 32, ld_relaxed_u64(keys + 32), p.ctrl) : 0ull;
  float lp = 0.0f;  // log2 p_i(x_i)
  if (lane < k) {
    float m, sm;
    unpack_stats(take(stats + lane, ld_relaxed_u64(stats + lane), p.ctrl), m, sm);
    const int x = __ldg(p.tokens + static_cast<size_t>(b) * k + lane);
    if (x >= 0 && x < V &&
        SV_IN(p.ctrl, static_cast<long long>(b) * p.sb + static_cast<long long>(lane) * p.sp + x,
              p.t_elems)) {
      const long long off = static_cast<long long>(b) * p.sb + static_cast<long long>(lane) * p.sp + x;
      const float l = p.t_dtype == 1 ? load_elem<uint16_t>(p.tgt, off) : load_elem<float>(p.tgt, off);
      lp = fmaf(l, p.c2, -m) - lg2f(sm);
    } else {
      lp = -INFINITY;
    }
  }
  float cum = lp;  // inclusive prefix sum over lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float up = __shfl_up_sync(0xffffffffu, cum, o);
    if (lane >= o) cum += up;
  }
  const bool fail = lane < k && !(cum >= p.log2_tau);
  const unsigned int mm = __ballot_sync(0xffffffffu, fail);
  const int n = mm ? __ffs(mm) - 1 : k;
  const int an = __shfl_sync(0xffffffffu, key_index(kv), n & 31);
  const int a32 = __shfl_sync(0xffffffffu, key_index(k32), 0);
  const int next = n == 32 ? a32 : an;
  int* out = p.out_tokens + static_cast<size_t>(b) * (k + 1);
  for (int i = lane; i <= k; i += 32)
    out[i] = i < n ? __ldg(p.tokens + static_cast<size_t>(b) * k + i) : (i == n ? next : -1);
  if (lane == 0) {
    p.accepted_len[b] = n;
    p.seq[b].cnt1 = 0u;
  }
}

// Tree form of the finalize (one warp; nodes j = lane and lane + 32): from
// the root, step to the lowest-index child whose token equals the current
// node's row argmax, until none does; commit the path's tokens and the last
// node's argmax.  Row keys are read without clearing and cleared at the end.
__device__ void finalize_argmax_tree(const ArgmaxParams& p, int b, int lane) {
  const int N = p.R;
  unsigned long long* keys = p.rkey + static_cast<size_t>(b) * N;
  for (int r = lane; r < N; r += 32)
    if (ld_relaxed_u64(keys + r) == 0ull) poll_u64(keys + r, p.ctrl);  // published by now
  __syncwarp();
  const int* par = p.parent + static_cast<size_t>(b) * N;
  const int* tok = p.tokens + static_cast<size_t>(b) * N;
  int a[2], pj[2], tj[2];
  bool bad = false;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = lane + 32 * h;
    a[h] = j < N ? key_index(ld_relaxed_u64(keys + j)) : -1;
    pj[h] = -1;
    tj[h] = -1;
    if (j >= 1 && j < N) {
      const int q = __ldg(par + j);
      if (q >= 0 && q < j) {
        pj[h] = q;
        tj[h] = __ldg(tok + j);
      } else {
        bad = true;  // never entered
      }
    }
  }
  int* path = p.path + static_cast<size_t>(b) * N;
  int* out = p.out_tokens + static_cast<size_t>(b) * N;
  // every step enters a child c > u (parents precede their children), so the
  // walk ends within N - 1 steps
  int u = 0, n = 0, au;
  for (;;) {
    au = __shfl_sync(0xffffffffu, u < 32 ? a[0] : a[1], u & 31);
    const unsigned int m0 = __ballot_sync(0xffffffffu, pj[0] == u && tj[0] == au);
    const unsigned int m1 = __ballot_sync(0xffffffffu, pj[1] == u && tj[1] == au);
    if (m0 == 0u && m1 == 0u) break;
    const int c = m0 ? __ffs(m0) - 1 : 32 + __ffs(m1) - 1;
    const int tc = __shfl_sync(0xffffffffu, c < 32 ? tj[0] : tj[1], c & 31);
    if (lane == 0) {
      path[n + 1] = c;
      out[n] = tc;
    }
    u = c;
    ++n;
  }
  if (lane == 0) {
    path[0] = 0;
    out[n] = au;  // the target's extra token
  }
  for (int j = n + 1 + lane; j < N; j += 32) {
    path[j] = -1;
    out[j] = -1;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&p.ctrl->flags, kFlagInvalidTree);
  __syncwarp();
  for (int r = lane; r < N; r += 32) keys[r] = 0ull;
  if (lane == 0) {
    p.accepted_len[b] = n;
    p.seq[b].cnt1 = 0u;
  }
}

// Rows form of the finalize: the row keys of sequence b are read without
// clearing (several (g, i) may share a row), looked up through row_of, and
// cleared at the end.
__device__ void finalize_argmax_rows(const ArgmaxParams& p, int b, int lane) {
  const int k = p.k, G = p.G, R = p.R;
  unsigned long long* keys = p.rkey + static_cast<size_t>(b) * R;
  for (int r = lane; r < R; r += 32)
    if (ld_relaxed_u64(keys + r) == 0ull) poll_u64(keys + r, p.ctrl);  // published by now
  __syncwarp();
  const int* map = p.row_of + static_cast<size_t>(b) * G * (k + 1);
  int best_n = -1, best_g = 0, best_next = -1;
  bool bad = false;
  for (int g = 0; g < G; ++g) {
    // a[i] for i = lane and i = lane + 32 (k + 1 <= 33 rows per branch)
    int a[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = lane + 32 * h;
      a[h] = -1;
      if (i <= k) {
        const int r = __ldg(map + g * (k + 1) + i);
        if (r >= 0 && r < R) {
          a[h] = key_index(ld_relaxed_u64(keys + r));
        } else {
          bad = true;
        }
      }
    }
    const int* cand = p.tokens + (static_cast<size_t>(b) * G + g) * k;
    const bool miss = lane < k && __ldg(cand + lane) != a[0];
    const unsigned int mm = __ballot_sync(0xffffffffu, miss);
    const int n = mm ? __ffs(mm) - 1 : k;
    const int an = __shfl_sync(0xffffffffu, a[0], n & 31);
    const int a32 = __shfl_sync(0xffffffffu, a[1], 0);
    if (n > best_n) {
      best_n = n;
      best_g = g;
      best_next = (n == 32) ? a32 : an;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&p.ctrl->flags, kFlagInvalidRow);
  const int* cand = p.tokens + (static_cast<size_t>(b) * G + best_g) * k;
  int* out = p.out_tokens + static_cast<size_t>(b) * (k + 1);
  for (int i = lane; i <= k; i += 32)
    out[i] = i < best_n ? __ldg(cand + i) : (i == best_n ? best_next : -1);
  __syncwarp();
  for (int r = lane; r < R; r += 32) keys[r] = 0ull;
  if (lane == 0) {
    p.accepted_len[b] = best_n;
    if (p.best_g) p.best_g[b] = best_g;
    p.seq[b].cnt1 = 0u;
  }
}

// Finalize of sequence b (one warp): per branch, the accepted length is the
// first position whose draft differs from the row argmax (ballot); the
// longest branch (lowest g on a tie) is committed.
// kOneGrid: called by the finalize grid of the one-grid path, which runs after
// the streaming grid has completed; no branch state to clear, so no fence.
#ifndef SV_FIN_BRANCHES
#define SV_FIN_BRANCHES 8
#endif
constexpr int kFinBranches = SV_FIN_BRANCHES;  // branches whose loads go out together
template <bool kOneGrid>
__device__ void finalize_argmax(const ArgmaxParams& p, int b, int lane) {
  const int k = p.k, G = p.G;
  unsigned long long* keys = p.rkey + static_cast<size_t>(b) * G * (k + 1);
  int best_n = -1, best_g = 0, best_next = -1;
  bool invalid = false;  // a draft token outside [0, V): it never matches
  for (int g0 = 0; g0 < G; g0 += kFinBranches) {
    // row keys and draft tokens of up to kFinBranches branches: loads issued
    // together, the tokens (inputs) before any key is examined
    unsigned long long v[kFinBranches], v32[kFinBranches];
    int xs[kFinBranches];
#pragma unroll
    for (int q = 0; q < kFinBranches; ++q) {
      const int g = g0 + q;
      v[q] = (g < G && lane <= k) ? ld_relaxed_u64(keys + g * (k + 1) + lane) : 0ull;
      v32[q] = (g < G && k == 32 && lane == 0) ? ld_relaxed_u64(keys + g * (k + 1) + 32) : 0ull;
      xs[q] = (g < G && lane < k) ? __ldg(p.tokens + (static_cast<size_t>(b) * G + g) * k + lane)
                                  : 0;
    }
#pragma unroll
    for (int q = 0; q < kFinBranches; ++q) {
      const int g = g0 + q;
      if (g >= G) break;
      const int a = lane <= k ? key_index(take(keys + g * (k + 1) + lane, v[q], p.ctrl)) : -1;
      const int a32 =
          (k == 32 && lane == 0) ? key_index(take(keys + g * (k + 1) + 32, v32[q], p.ctrl)) : -1;
      const int x = xs[q];
      invalid |= x < 0 || x >= p.V;
      const bool miss = lane < k && x != a;
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
  }
  if (__any_sync(0xffffffffu, invalid) && lane == 0) atomicOr(&p.ctrl->flags, kFlagInvalidToken);
  if (!kOneGrid && lane == 0) {
    // acquire (this lane counted the last row): every branch-state update
    // lands before the clear
    fence_acq_rel_gpu();
    for (int g = 0; g < G; ++g) p.dead[static_cast<size_t>(b) * G + g] = 0u;
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

// Row merge (one warp, one lane per chunk): the row's argmax key is the
// largest chunk key; count the row, and the last row finalizes.
template <int kMode>
__device__ void merge_argmax_row(const ArgmaxParams& p, int b, int r, int lane) {
  const unsigned int R = static_cast<unsigned int>(p.R);
  if (!SV_IN(p.ctrl, b, p.B) || !SV_IN(p.ctrl, r, p.R)) return;
  unsigned long long* slot = p.slots + (static_cast<size_t>(b) * R + r) * p.nch;
  unsigned long long key = 0ull;
  for (int c = lane; c < p.nch; c += 32) {
    const unsigned long long v = take(slot + c, ld_relaxed_u64(slot + c), p.ctrl);
    key = v > key ? v : key;
  }
  key = warp_max_u64(key);
  const bool with_stats = kMode == kArgThreshold && r < p.k;
  float M = -INFINITY, S = 0.0f;
  if (with_stats) {
    unsigned long long* ss = p.sslots + (static_cast<size_t>(b) * R + r) * p.nch;
    for (int c = lane; c < p.nch; c += 32) {
      float m, sv;
      unpack_stats(take(ss + c, ld_relaxed_u64(ss + c), p.ctrl), m, sv);
      merge_stats(M, S, m, sv);
    }
    const float4 w = warp_stats2(make_float4(M, S, -INFINITY, 0.0f));
    M = w.x;
    S = w.y;
  }
  unsigned int old = 0u;
  if (lane == 0) {
    if (kMode == kArgPlain) {
      // a draft that differs from this row's argmax ends its branch here:
      // later rows of the branch decide nothing
      const int g = r / (p.k + 1), pos = r - g * (p.k + 1);
      if (pos < p.k &&
          __ldg(p.tokens + (static_cast<size_t>(b) * p.G + g) * p.k + pos) != key_index(key)) {
        atomicMax(p.dead + static_cast<size_t>(b) * p.G + g, 64u - static_cast<unsigned int>(pos));
        // the finalize, which clears the word, sees this update before the
        // row count below (a fence: a release operation would order only
        // what came before it)
        fence_acq_rel_gpu();
      }
    }
    if (with_stats) st_relaxed_u64(p.rstats + static_cast<size_t>(b) * R + r, pack_stats(M, S));
    st_relaxed_u64(p.rkey + static_cast<size_t>(b) * R + r, key);
    p.rc[static_cast<size_t>(b) * R + r] = 0u;
    old = atomicAdd(&p.seq[b].cnt1, 1u);
  }
  if (__shfl_sync(0xffffffffu, old == R - 1u ? 1 : 0, 0)) {
    if constexpr (kMode == kArgThreshold)
      finalize_threshold(p, b, lane);
    else if constexpr (kMode == kArgTree)
      finalize_argmax_tree(p, b, lane);
    else if constexpr (kMode == kArgRows)
      finalize_argmax_rows(p, b, lane);
    else
      finalize_argmax<false>(p, b, lane);
  }
}

template <int kMode>
__device__ void argmax_epilogue(const ArgmaxParams& p, Shared& sh, int group, int lane) {
  const unsigned int R = static_cast<unsigned int>(p.R);
  const unsigned int last = static_cast<unsigned int>(p.nch) - 1u;
  int pend_b = -1, pend_r = 0;  // unresolved arrival (sequence, row), or -1
  unsigned int pend_old = 0u;
  for (uint32_t use = group;; use += kComputeGroups) {
    const int s = use % kStages;
    const uint32_t parity = (use / kStages) & 1u;
    if (pend_b >= 0 && !mbar_try_wait(&sh.rfull[s], parity)) {
      if (__shfl_sync(0xffffffffu, pend_old == last ? 1 : 0, 0))
        merge_argmax_row<kMode>(p, pend_b, pend_r, lane);
      pend_b = -1;
    }
    if (!mbar_wait(&sh.rfull[s], parity, p.ctrl)) break;
    const Hdr h = sh.hdr[s];
    if (h.kind == kKindEnd) break;
    if (h.kind == kKindRowDone) {  // every chunk of the row is counted: merge it
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.empty[s]);
      if (pend_b >= 0 && __shfl_sync(0xffffffffu, pend_old == last ? 1 : 0, 0))
        merge_argmax_row<kMode>(p, pend_b, pend_r, lane);
      pend_b = -1;
      merge_argmax_row<kMode>(p, h.b, h.i, lane);
      continue;
    }
    float v = -INFINITY;
    int i = INT_MAX;
    float4 st = make_float4(-INFINITY, 0.0f, -INFINITY, 0.0f);
    if (lane < kGroupWarps) {
      const float4 r = sh.res[s][lane];
      v = r.x;
      i = __float_as_int(r.y);
      st.x = r.z;
      st.y = r.w;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.empty[s]);
    if (!SV_IN(p.ctrl, h.b, p.B) || !SV_IN(p.ctrl, h.i, p.R) || !SV_IN(p.ctrl, h.c, p.nch))
      continue;
    warp_argmax(v, i);
    const bool with_stats = kMode == kArgThreshold && h.i < p.k;
    if (with_stats) st = warp_stats2(st);
    unsigned int old = 0u;
    if (lane == 0) {
      const size_t slot = (static_cast<size_t>(h.b) * R + h.i) * p.nch + h.c;
      st_relaxed_u64(p.slots + slot, make_key(v, i));
      if (with_stats) st_relaxed_u64(p.sslots + slot, pack_stats(st.x, st.y));
      old = atomicAdd(&p.rc[static_cast<size_t>(h.b) * R + h.i], 1u);
    }
    if (pend_b >= 0 && __shfl_sync(0xffffffffu, pend_old == last ? 1 : 0, 0))
      merge_argmax_row<kMode>(p, pend_b, pend_r, lane);
    pend_b = h.b;
    pend_r = h.i;
    pend_old = old;
  }
  if (pend_b >= 0 && __shfl_sync(0xffffffffu, pend_old == last ? 1 : 0, 0))
    merge_argmax_row<kMode>(p, pend_b, pend_r, lane);
}

template <typename TT, bool kTma, int kMode>
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
      mbar_init(&sh.rfull[s], kGroupWarps);
    }
    mbar_fence_init();
  }
  __syncthreads();
  dep_enter();
  if (warp < kProducerWarps) {
    if (lane == 0 && warp < kArgmaxProducers)
      argmax_producer<TT, kTma, kMode == kArgRows || kMode == kArgTree, kMode == kArgPlain>(
          p, sh, stages, kArgmaxProducers == 1 ? -1 : warp);
  } else if (warp < kProducerWarps + kComputeWarps) {
    argmax_compute<TT, kTma, kMode>(p, sh, stages, warp - kProducerWarps, lane);
  } else {
    argmax_epilogue<kMode>(p, sh, warp - kProducerWarps - kComputeWarps, lane);
  }
}

// ========================================================= one-shot argmax

// Plain greedy and multi-candidate verify for calls too small for the
// persistent pipeline to pay off (a few microseconds of ramp and a dependent
// tail of several L2 round trips after the last chunk, against a call of a
// few tens of microseconds, and too short for a rejection to be known before
// the rows after it are read).  One 256-thread block per chunk of one row
// (16 KB; 8 KB and 32 KB chunks measured slower, 26.0 and 21.9 against
// 19.8 us at B = 64, k = 4, V = 128256): every thread loads its (up to) four
// 16-byte vectors at once and takes the first maximum, the block merges its
// warps in shared memory and publishes the chunk's key with one 64-bit
// atomicMax on the row key (keys order like (value, -index), so the max is
// the row's first maximum), whose result it does not wait for, and exits.
// A block that also counted itself and let the last block of its sequence
// finalize held its slot on the SM for two more L2 round trips, a third of
// its life, and the resident blocks are what keeps bytes in flight.  So a
// second grid of one warp per sequence runs the same finalize as the
// persistent kernel; it is launched as a programmatic dependent of the
// first, so its launch overlaps the streaming, and its griddepcontrol.wait
// returns once the first grid has completed and its atomics are visible.
#ifndef SV_OS_THREADS
#define SV_OS_THREADS 256
#endif
#ifndef SV_OS_VECS
#define SV_OS_VECS 4
#endif
constexpr int kOsThreads = SV_OS_THREADS;
constexpr int kOsVecs = SV_OS_VECS;

template <typename T>
__host__ __device__ constexpr int oneshot_chunk() {
  return kOsThreads * kOsVecs * Elem<T>::kPerVec;  // 8192 bf16 or 4096 f32 entries
}

int oneshot_chunk_entries(int t_dtype) {
  return t_dtype == 1 ? oneshot_chunk<uint16_t>() : oneshot_chunk<float>();
}

// Largest key of chunk `ch` (row b * R + r, column chunk c) over the block;
// returned in thread 0 (0 for a chunk with no finite-or-infinite entry).
template <typename T, bool kVec>
__device__ __forceinline__ unsigned long long oneshot_chunk_key(const ArgmaxParams& p,
                                                                unsigned int ch, int tid,
                                                                unsigned long long* s_key,
                                                                unsigned int& row_out) {
  constexpr int EPV = Elem<T>::kPerVec;
  constexpr int CH = oneshot_chunk<T>();
  const int lane = tid & 31;
  const unsigned int row = udiv(ch, p.div_nch1);  // b * R + r
  const int c = static_cast<int>(ch - row * static_cast<unsigned int>(p.nch1));
  const unsigned int bu = udiv(row, p.div_R);
  const int b = static_cast<int>(bu);
  const int r = static_cast<int>(row - bu * static_cast<unsigned int>(p.R));
  const int g = r / (p.k + 1), pos = r - g * (p.k + 1);
  const long long off = static_cast<long long>(b) * p.sb + static_cast<long long>(g) * p.sg +
                        static_cast<long long>(pos) * p.sp;
  const int x0 = c * CH;
  int len = min(CH, p.V - x0);
  if (!SV_IN(p.ctrl, b, p.B) || !SV_IN_RANGE(p.ctrl, off + x0, len, p.t_elems)) len = 0;
  float best = -INFINITY;
  int idx = INT_MAX;
  if (kVec) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.tgt) + off + x0);
    const int nv = len / EPV;
    uint4 v[kOsVecs];
#pragma unroll
    for (int q = 0; q < kOsVecs; ++q) {
      const int i = tid + q * kOsThreads;
      v[q] = i < nv ? __ldcs(src + i) : neg_inf_vec<T>();  // read once: streaming hint
    }
    int bj = -1;
    uint4 bvec = v[0];
#pragma unroll
    for (int q = 0; q < kOsVecs; ++q) {  // increasing index: the first maximum is kept
      const float m = vec_max<T>(v[q]);
      const bool take = tid + q * kOsThreads < nv && (bj < 0 || m > best);
      best = take ? m : best;
      bj = take ? q : bj;
      bvec = take ? v[q] : bvec;
    }
    if (bj >= 0) {
      float f[EPV];
      unpack(bvec, f);
      const int x = x0 + (tid + bj * kOsThreads) * EPV;
#pragma unroll
      for (int q = EPV - 1; q >= 0; --q)
        if (f[q] == best) idx = x + q;
    }
    const int e = nv * EPV + tid;  // the ragged end is shorter than one vector
    if (e < len) {
      const float t = load_elem<T>(p.tgt, off + x0 + e);
      if (better(t, x0 + e, best, idx)) {
        best = t;
        idx = x0 + e;
      }
    }
  } else {
    for (int e = tid; e < len; e += kOsThreads) {
      const float t = load_elem<T>(p.tgt, off + x0 + e);
      if (better(t, x0 + e, best, idx)) {
        best = t;
        idx = x0 + e;
      }
    }
  }
  warp_argmax(best, idx);
  if (lane == 0) s_key[tid >> 5] = idx == INT_MAX ? 0ull : make_key(best, idx);
  __syncthreads();
  unsigned long long key = 0ull;
  if (tid == 0) {
#pragma unroll
    for (int w = 0; w < kOsThreads / 32; ++w) key = s_key[w] > key ? s_key[w] : key;
  }
  row_out = row;
  return key;
}

// Blocks take chunks blockIdx.x, + gridDim.x, ... (one each when the grid
// covers every chunk).  The warp keys alternate between two shared arrays,
// so one barrier a chunk suffices: thread 0 has read a chunk's array before
// it passes the next chunk's barrier, and the array is written again only
// after that.
template <typename T, bool kVec>
__global__ void __launch_bounds__(kOsThreads)
    argmax_oneshot_kernel(const __grid_constant__ ArgmaxParams p) {
  __shared__ unsigned long long s_key[2][kOsThreads / 32];
  // (the finalize grid may then be scheduled once every block has started;
  // it still waits for this grid to complete)
  dep_enter();
  const int tid = threadIdx.x;
  const unsigned int total =
      static_cast<unsigned int>(p.B) * static_cast<unsigned int>(p.R) * static_cast<unsigned int>(p.nch1);
  int par = 0;
  for (unsigned int ch = blockIdx.x; ch < total; ch += gridDim.x, par ^= 1) {
    unsigned int row;
    const unsigned long long key = oneshot_chunk_key<T, kVec>(p, ch, tid, s_key[par], row);
    if (tid == 0 && key && SV_IN(p.ctrl, row, static_cast<long long>(p.B) * p.R))
      atomicMax(p.rkey + row, key);  // result unused: a fire-and-forget reduction
  }
}

// One warp per sequence, once every block of the streaming grid has published
// its key (griddepcontrol.wait: that grid has completed and its atomics are
// visible).
__global__ void __launch_bounds__(256) argmax_finalize_kernel(const __grid_constant__ ArgmaxParams p) {
  const int b = static_cast<int>(blockIdx.x) * 8 + (static_cast<int>(threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  // The draft tokens are inputs, complete before the streaming grid began:
  // bring this sequence's into L2 while that grid still runs.
  if (b < p.B) {
    const char* tok = reinterpret_cast<const char*>(p.tokens + static_cast<size_t>(b) * p.G * p.k);
    const int bytes = p.G * p.k * static_cast<int>(sizeof(int));
    for (int o = lane * 128; o < bytes; o += 32 * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(tok + o));
  }
  dep_enter();
  if (b < p.B) {
    if (p.row_of)
      finalize_argmax_rows(p, b, lane);
    else
      finalize_argmax<true>(p, b, lane);
  }
}

template <typename T>
static cudaError_t launch_oneshot_t(const ArgmaxParams& p, bool vec, cudaStream_t st) {
  const long long blocks = static_cast<long long>(p.B) * p.R * p.nch1;
  if (blocks <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned int>(blocks));
  cudaError_t e = counted(
      vec ? launch_k(SV_PDL >= 2, argmax_oneshot_kernel<T, true>, grid, dim3(kOsThreads), 0, st, p)
          : launch_k(SV_PDL >= 2, argmax_oneshot_kernel<T, false>, grid, dim3(kOsThreads), 0, st,
                     p),
      1);
  if (e != cudaSuccess) return e;
  // launched while the streaming grid runs; its warps wait for that grid
  return counted(launch_k(SV_PDL >= 1, argmax_finalize_kernel,
                          dim3(static_cast<unsigned int>((p.B + 7) / 8)), dim3(256), 0, st, p),
                 1);
}

cudaError_t launch_argmax_oneshot(const ArgmaxParams& p, int t_dtype, bool vec, cudaStream_t st) {
  return t_dtype == 1 ? launch_oneshot_t<uint16_t>(p, vec, st) : launch_oneshot_t<float>(p, vec, st);
}

// ================================================================ philox

__global__ void philox_kernel(const uint4* __restrict__ ctr, long long n, uint32_t k0,
                              uint32_t k1, uint4* __restrict__ out) {
  dep_enter();
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < n;
       j += static_cast<long long>(gridDim.x) * blockDim.x)
    out[j] = philox10(ctr[j], k0, k1);
}

// ================================================================ commit

// One warp per sequence: lane 0 reads the length, every lane copies up to two
// of the n + 1 committed tokens (k + 1 <= 33), then lane 0 advances the
// length and writes the next input.
__global__ void commit_kernel(const int* __restrict__ accepted_len,
                              const int* __restrict__ out_tokens, int B, int k,
                              int* __restrict__ seq_len, int* __restrict__ token_buf,
                              long long buf_stride, int capacity, int* __restrict__ next_input,
                              Ctrl* ctrl) {
  dep_enter();
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const int n = min(max(__ldg(accepted_len + b), 0), k);
  const int L = max(seq_len[b], 0);
  const int* out = out_tokens + static_cast<size_t>(b) * (k + 1);
  int* buf = token_buf + static_cast<size_t>(b) * buf_stride;
  bool full = false;
  for (int j = lane; j <= n; j += 32) {
    const long long pos = static_cast<long long>(L) + j;
    if (pos < capacity)
      buf[pos] = __ldg(out + j);
    else
      full = true;
  }
  full = __any_sync(0xffffffffu, full);
  if (lane == 0) {
    const long long end = static_cast<long long>(L) + n + 1;
    seq_len[b] = static_cast<int>(end < capacity ? end : capacity);
    if (next_input) next_input[b] = __ldg(out + n);
    if (full && ctrl) atomicOr(&ctrl->flags, kFlagCapacity);
  }
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
  return counted(launch_k(SV_PDL >= 2, kernel, dim3(grid), dim3(kThreads), smem, st, p), 1);
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

template <typename TT, bool kTma, int kMode>
static cudaError_t launch_argmax_t(const ArgmaxParams& p, int grid, size_t smem, cudaStream_t st) {
  static bool done[64] = {};
  auto kernel = argmax_verify_kernel<TT, kTma, kMode>;
  cudaError_t e = prepare(kernel, smem, done);
  if (e != cudaSuccess) return e;
  return counted(launch_k(SV_PDL >= 2, kernel, dim3(grid), dim3(kThreads), smem, st, p), 1);
}

template <typename TT>
static cudaError_t launch_argmax_mode(const ArgmaxParams& p, int mode, bool tma, int grid,
                                      size_t smem, cudaStream_t st) {
  switch (mode) {
    case kArgRows:
      return tma ? launch_argmax_t<TT, true, kArgRows>(p, grid, smem, st)
                 : launch_argmax_t<TT, false, kArgRows>(p, grid, smem, st);
    case kArgTree:
      return tma ? launch_argmax_t<TT, true, kArgTree>(p, grid, smem, st)
                 : launch_argmax_t<TT, false, kArgTree>(p, grid, smem, st);
    case kArgThreshold:
      return tma ? launch_argmax_t<TT, true, kArgThreshold>(p, grid, smem, st)
                 : launch_argmax_t<TT, false, kArgThreshold>(p, grid, smem, st);
    default:
      return tma ? launch_argmax_t<TT, true, kArgPlain>(p, grid, smem, st)
                 : launch_argmax_t<TT, false, kArgPlain>(p, grid, smem, st);
  }
}

cudaError_t launch_argmax(const ArgmaxParams& p, int t_dtype, bool tma, int grid, size_t smem,
                          cudaStream_t st) {
  const int mode = p.sslots ? kArgThreshold : p.parent ? kArgTree : p.row_of ? kArgRows : kArgPlain;
  return t_dtype == 1 ? launch_argmax_mode<uint16_t>(p, mode, tma, grid, smem, st)
                      : launch_argmax_mode<float>(p, mode, tma, grid, smem, st);
}

cudaError_t launch_commit(const int* accepted_len, const int* out_tokens, int B, int k,
                          int* seq_len, int* token_buf, long long buf_stride, int capacity,
                          int* next_input, Ctrl* ctrl, cudaStream_t st) {
  if (B <= 0) return cudaSuccess;
  constexpr int kWarps = 8;
  return counted(launch_k(SV_PDL >= 2, commit_kernel, dim3((B + kWarps - 1) / kWarps),
                          dim3(32 * kWarps), 0, st, accepted_len, out_tokens, B, k, seq_len,
                          token_buf, buf_stride, capacity, next_input, ctrl),
                 1);
}

cudaError_t launch_philox(const uint4* ctr, long long n, unsigned int key0, unsigned int key1,
                          uint4* out, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const long long blocks = (n + 255) / 256;
  const int grid = static_cast<int>(blocks < 4096 ? blocks : 4096);
  return counted(
      launch_k(SV_PDL >= 2, philox_kernel, dim3(grid), dim3(256), 0, st, ctr, n, key0, key1, out),
      1);
}

}  // namespace sv
