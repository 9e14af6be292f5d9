// Pieces shared by the two decode kernels (CUDA-core and tensor-core):
// kernel parameters, the balanced work partition over persistent CTAs, and
// the merge of split units through the workspace.
//
// Work partition.  Each (sequence, kv head) "unit" is cut into granules of
// CB consecutive logical blocks (the last one may be shorter).  CB is the
// kernel's processing chunk (1 block for the CUDA-core kernel, 8 for the
// tensor-core kernel).  Every unit is given a cost: kGranuleCost per granule
// plus `unit_cost` for the fixed work of finishing a unit (sums, output or
// partial state, merge).  The units are laid end to end on a cost line —
// sequence-major, kv head next — each as its fixed cost followed by its
// granules, and the line is cut into `nparts` contiguous ranges of equal
// cost, one per CTA.  A CTA processes the granules that start in its range,
// so CTAs get equal expected time whatever the mix of unit lengths, and no
// range boundary splits a chunk.  nparts is the grid size, or fewer when
// there is less than one granule of cost per CTA, so that every range that
// falls inside a unit holds one of its granules.  A CTA's granules fall into
// segments, one per unit it touches.  A unit covered by one CTA is finished
// there.  A unit split between CTAs is merged in the same launch: by
// whichever CTA arrives last (finish_split_unit, the CUDA-core kernel), or
// by the CTA holding the unit's first piece (the tensor-core kernels).
//
// Merge rule (study notes ch.05 §4, the online-softmax merge applied to
// partitions): a partial state is (m, l, acc) in the log2 domain — running
// max m, sum l of 2^(score - m), unnormalised output acc.  Combining states
// rescales each by 2^(m_p - M) with M = max m_p; out = sum acc' / sum l'.
#pragma once

#include <cstdint>

#include "pa_device.cuh"

namespace pa {

struct DecodeParams {
  const uint16_t* q;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  uint16_t* out;
  float* partials;
  int32_t* counters;
  int32_t* status;
  int max_nb;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int num_blocks;
  float scale_log2;
  unsigned long long wait_limit_ns;
  int test_flags;
  // multi-query decode: query positions per sequence (q, out are
  // [num_seqs][q_len][num_q_heads][head_dim]); 1 otherwise
  int q_len;
  // multi-query decode: row tiles per sequence (a unit carries the positions
  // of one tile); 1 otherwise
  int q_tiles;
  // shared-prefix decode (null / 0 otherwise)
  const int32_t* group_starts;   // [num_groups + 1], consecutive sequences per group
  const int32_t* group_prefix;   // [num_groups] shared leading blocks of each group
  int num_groups;
  // partition cost of finishing a unit, in 1/kGranuleCost granules
  int unit_cost;
  // new tokens' K/V stored by the tensor-core kernel before it reads the
  // pools (null / 0 for none), the phase closed by a grid-wide barrier whose
  // two words sit at grid_sync in the workspace
  const uint4* upd_k;         // [upd_num_tokens][num_kv_heads][head_dim]
  const uint4* upd_v;
  const int64_t* upd_slots;   // [upd_num_tokens]
  int upd_num_tokens;
  int32_t* grid_sync;
  // per output row (num_q_heads per sequence row), the natural log of the
  // softmax normaliser, log sum_t exp(scale q.K_t); -inf for no token.
  // Written by the tensor-core kernel when not null.
  float* lse;
};

// Workspace bytes of the grid-wide barrier's words (one 128-byte line used),
// between the partial states and the arrival counters.
constexpr int kGridSyncBytes = 256;

constexpr long long kGranuleCost = 8;  // partition cost of one granule

constexpr int kFlagTestWithholdCopies = PA_DECODE_TEST_WITHHOLD_COPIES;  // producer issues nothing
constexpr int kFlagTestSkipUpdateArrival = PA_DECODE_TEST_SKIP_UPDATE_ARRIVAL;  // CTA 0 skips the stores' barrier

__device__ __forceinline__ int checked_len(const DecodeParams& p, int s, int B) {
  const int n = __ldg(p.seq_lens + s);
  return (n < 0 || n > p.max_nb * B) ? 0 : n;
}

// The blocks a "sequence" of the work list covers: logical blocks
// [first, nb) of a sequence of len tokens.  The default span is the whole
// sequence; other kernels cover only a suffix, or a group's shared prefix.
struct SeqSpan {
  int first, nb, len;
};

struct WholeSequence {
  template <int B>
  __device__ __forceinline__ SeqSpan span(const DecodeParams& p, int s) const {
    const int len = checked_len(p, s, B);
    return SeqSpan{0, (len + B - 1) / B, len};
  }
  __device__ __forceinline__ int count(const DecodeParams& p) const { return p.num_seqs; }
};

struct Cursor {
  int s, h;
  int jg;     // next granule of unit (s, h)
  int ng;     // granules of sequence s's units
  int first;  // first logical block of the span
  int nb;     // end of the span (logical blocks)
  int len;    // tokens of sequence s
  long long ucost;  // cost-line position where unit (s, h) starts
  long long end;    // end of the CTA's cost range
  bool done;
};

struct Seg {
  int s, h;
  int j0, n;  // logical blocks [j0, j0 + n) of unit (s, h)
  int first;  // first logical block of the unit's span
  int nb;     // end of the unit's span
  int ng;     // granules of the unit
  int len;    // tokens of the sequence
  long long unit_first;  // cost-line position of the unit's granule 0
  long long unit_last;   // cost-line position of its last granule
};

// Cost of one unit with ng granules (a unit with none costs nothing).
__device__ __forceinline__ long long unit_cost_of(const DecodeParams& p, int ng) {
  return ng > 0 ? ng * kGranuleCost + p.unit_cost : 0;
}

template <int B, int CB, class Src>
__device__ __forceinline__ void load_seq(Cursor& c, const DecodeParams& p, const Src& src) {
  const SeqSpan sp = src.template span<B>(p, c.s);
  c.len = sp.len;
  c.first = sp.first;
  c.nb = sp.nb;
  c.ng = sp.nb > sp.first ? (sp.nb - sp.first + CB - 1) / CB : 0;
}

// Move the cursor to granule 0 of the next unit that has one.
template <int B, int CB, class Src>
__device__ __forceinline__ void next_unit(Cursor& c, const DecodeParams& p, const Src& src) {
  c.ucost += unit_cost_of(p, c.ng);
  c.jg = 0;
  if (++c.h == p.num_kv_heads) {
    c.h = 0;
    do {
      if (++c.s >= src.count(p)) {  // past the last sequence
        c.done = true;
        break;
      }
      load_seq<B, CB>(c, p, src);
    } while (c.ng == 0);
  }
}

// Next segment of the CTA's range (the granules of one unit that start in
// it); advances the cursor past it.
template <int B, int CB, class Src = WholeSequence>
__device__ __forceinline__ bool next_seg(Cursor& c, Seg& sg, const DecodeParams& p, const Src& src = Src()) {
  if (c.done) return false;
  const long long g0 = c.ucost + p.unit_cost + c.jg * kGranuleCost;  // where granule jg starts
  if (g0 >= c.end) {
    c.done = true;
    return false;
  }
  const long long fit = (c.end - g0 + kGranuleCost - 1) / kGranuleCost;  // granules starting before end
  const int k = static_cast<int>(fit < c.ng - c.jg ? fit : c.ng - c.jg);
  sg.s = c.s;
  sg.h = c.h;
  sg.j0 = c.first + c.jg * CB;
  const int j1 = c.first + (c.jg + k) * CB;
  sg.n = (j1 < c.nb ? j1 : c.nb) - sg.j0;
  sg.first = c.first;
  sg.nb = c.nb;
  sg.ng = c.ng;
  sg.len = c.len;
  sg.unit_first = c.ucost + p.unit_cost;
  sg.unit_last = sg.unit_first + (c.ng - 1) * kGranuleCost;
  c.jg += k;
  if (c.jg == c.ng) next_unit<B, CB>(c, p, src);
  return true;
}

// CTA whose range [c*N/C, (c+1)*N/C) of the cost line holds position x.
__device__ __forceinline__ long long cta_of(long long x, long long N, long long C) { return ((x + 1) * C - 1) / N; }

__device__ __forceinline__ long long range_start(long long c, long long N, long long C) { return c * N / C; }

struct RangeSmem {
  long long scan[32];
  long long pre0;
  int s0;
  int found;
};

// Block-wide inclusive scan of one value per thread (NT threads, all call).
template <int NT>
__device__ __forceinline__ long long block_inclusive_scan(long long v, RangeSmem& rs, long long& block_total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) rs.scan[warp] = v;
  __syncthreads();
  long long before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const long long t = rs.scan[w];
    if (w < warp) before += t;
    total += t;
  }
  __syncthreads();
  block_total = total;
  return v + before;
}

struct WorkRange {
  long long total;   // length of the cost line
  long long nparts;  // CTAs that own a range
  long long start, end;
};

// Every thread of the CTA calls this.  Writes zero outputs of empty
// sequences (each by one CTA), computes this CTA's range and positions the
// cursor at its first block.  Returns false when the CTA has no work.
template <int NT, int B, int CB, class Src = WholeSequence>
__device__ bool decode_prologue(const DecodeParams& p, RangeSmem& rs, WorkRange& wr, Cursor& cur,
                                const Src& src = Src()) {
  const int tid = threadIdx.x;
  const long long nctas = gridDim.x, cta = blockIdx.x;
  const int Hkv = p.num_kv_heads;
  const int nseq = src.count(p);
  long long mine = 0;
  const int nloop = nseq > p.num_seqs ? nseq : p.num_seqs;
  for (int s = tid; s < nloop; s += NT) {
    if (s < p.num_seqs && cta == 0) {
      const int raw = __ldg(p.seq_lens + s);
      if (raw < 0 || raw > p.max_nb * B) record_status(p.status, PA_DEV_BAD_SEQ_LEN);
    }
    if (s < nseq) {
      const SeqSpan sp = src.template span<B>(p, s);
      mine += Hkv * unit_cost_of(p, sp.nb > sp.first ? (sp.nb - sp.first + CB - 1) / CB : 0);
    }
  }
  long long line;
  const long long incl0 = block_inclusive_scan<NT>(mine, rs, line);
  wr.total = line;
  const long long most = line / kGranuleCost;  // at least one granule of cost per range
  wr.nparts = most < nctas ? most : nctas;
  if (cta >= wr.nparts) return false;  // uniform across the CTA (also covers an empty line)
  wr.start = range_start(cta, wr.total, wr.nparts);
  wr.end = range_start(cta + 1, wr.total, wr.nparts);

  // locate the sequence whose costs hold `start`: with at most one sequence
  // per thread the scan above already holds every prefix sum
  if (tid == 0) rs.found = 0;
  __syncthreads();
  if (nseq <= NT) {
    if (mine > 0 && incl0 - mine <= wr.start && wr.start < incl0) {
      rs.s0 = tid;
      rs.pre0 = incl0 - mine;
      rs.found = 1;
    }
    __syncthreads();
  }
  long long base = 0;
  for (int chunk = 0; chunk < nseq && !rs.found; chunk += NT) {
    const int s = chunk + tid;
    long long cost = 0;
    if (s < nseq) {
      const SeqSpan sp = src.template span<B>(p, s);
      cost = Hkv * unit_cost_of(p, sp.nb > sp.first ? (sp.nb - sp.first + CB - 1) / CB : 0);
    }
    long long chunk_total;
    const long long incl = block_inclusive_scan<NT>(cost, rs, chunk_total);
    const long long excl = incl - cost;
    if (cost > 0 && base + excl <= wr.start && wr.start < base + incl) {
      rs.s0 = s;
      rs.pre0 = base + excl;
      rs.found = 1;
    }
    base += chunk_total;
    __syncthreads();
  }
  if (!rs.found) return false;  // only with lengths changing under the kernel
  cur.s = rs.s0;
  load_seq<B, CB>(cur, p, src);
  const long long ucost = unit_cost_of(p, cur.ng);
  const long long off = wr.start - rs.pre0;
  cur.h = static_cast<int>(off / ucost);
  cur.ucost = rs.pre0 + cur.h * ucost;
  const long long rem = off - cur.h * ucost - p.unit_cost;  // past the unit's fixed cost
  cur.jg = rem <= 0 ? 0 : static_cast<int>((rem + kGranuleCost - 1) / kGranuleCost);
  cur.end = wr.end;
  cur.done = false;
  if (cur.jg >= cur.ng) next_unit<B, CB>(cur, p, src);  // the range starts after the unit's last granule
  return true;
}

// Zero the outputs of sequences whose length is 0 (or invalid): sequence s
// is written by CTA s % gridDim.x.  Called by all NT threads of every CTA
// before any early return.
template <int NT, int B>
__device__ __forceinline__ void zero_empty_outputs(const DecodeParams& p, int D) {
  const long long nctas = gridDim.x, cta = blockIdx.x;
  for (int s = threadIdx.x; s < p.num_seqs; s += NT) {
    if ((s % nctas) != cta) continue;
    if (checked_len(p, s, B) != 0) continue;
    uint4* o = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(s) * p.num_q_heads * D);
    for (int i = 0; i < p.num_q_heads * D / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
  }
}

// Partial slot of CTA c for a unit whose granule 0 is flattened index F: slot 0
// if c's range starts inside the unit, else slot 1 (the unit where it ends).
__device__ __forceinline__ size_t partial_slot(long long c, long long F, const WorkRange& wr) {
  const int sl = (range_start(c, wr.total, wr.nparts) >= F) ? 0 : 1;
  return static_cast<size_t>(c) * 2 + sl;
}

// Called by the `nthreads` threads that own a split unit's partial after it
// is written and fenced: bumps the unit's arrival counter; the last arrival
// merges every partial of the unit and writes the output.  `sync` is a
// barrier over exactly those threads; `is_last` is a shared int.
template <bool kBf16, int D, int G, typename Sync>
__device__ void finish_split_unit(const DecodeParams& p, const Seg& sg, const WorkRange& wr, int ctid,
                                  int nthreads, int* is_last, Sync sync) {
  constexpr int kStride = G * (D + 2);
  const long long F = sg.unit_first;
  const long long first = cta_of(F, wr.total, wr.nparts);
  const long long last = cta_of(sg.unit_last, wr.total, wr.nparts);
  int32_t* counter = p.counters + static_cast<size_t>(sg.s) * p.num_kv_heads + sg.h;
  sync();
  if (ctid == 0) {
    const int prev = atomicAdd(counter, 1);
    *is_last = (prev == static_cast<int>(last - first));
  }
  sync();
  if (*is_last) {
    __threadfence();
    uint16_t* out_row =
        p.out + (static_cast<size_t>(sg.s) * p.num_q_heads + static_cast<size_t>(sg.h) * G) * D;
    for (int idx = ctid; idx < G * D / 2; idx += nthreads) {
      const int g = (2 * idx) / D, d = (2 * idx) % D;
      float M = -INFINITY;
      for (long long cc = first; cc <= last; ++cc) {
        const float* pp = p.partials + partial_slot(cc, F, wr) * kStride;
        M = fmaxf(M, __ldcg(pp + g));
      }
      float L = 0.f, a0 = 0.f, a1 = 0.f;
      for (long long cc = first; cc <= last; ++cc) {
        const float* pp = p.partials + partial_slot(cc, F, wr) * kStride;
        const float sc = fast_exp2(__ldcg(pp + g) - M);
        L = fmaf(__ldcg(pp + G + g), sc, L);
        const float2 av = __ldcg(reinterpret_cast<const float2*>(pp + 2 * G + g * D + d));
        a0 = fmaf(av.x, sc, a0);
        a1 = fmaf(av.y, sc, a1);
      }
      const float inv = 1.f / L;
      *reinterpret_cast<uint32_t*>(out_row + g * D + d) = pack2<kBf16>(a0 * inv, a1 * inv);
    }
    if (ctid == 0) *counter = 0;
  }
}

}  // namespace pa
