// pa_decode — paged decode attention for sm_100a.
//
// What it computes (vLLM blog §"关键细节" 2); PagedAttention study notes ch.05 §4):
//   out[s][h] = softmax(scale * q[s][h] . K^T) V over the seq_lens[s] tokens
//   of sequence s, K/V reached block by block through block_tables, the
//   softmax normalisation merged across blocks with a running max and sum.
//
// How (B200 design):
//   * Work list.  All (sequence, kv head, logical block) triples are laid end
//     to end — sequence-major, kv head next, block innermost — and cut into
//     gridDim.x equal contiguous ranges, one per persistent CTA (grid = SMs x
//     resident CTAs).  Every CTA gets the same number of 8 KB K+V tile pairs
//     whatever the length mix, so ragged batches and long sequences
//     (split-KV) are one mechanism.  Each CTA derives its range from
//     seq_lens on the device; the host never reads lengths.
//   * Producer warp: walks the range, resolves each block's physical id once
//     (32 table entries per coalesced load), and issues one 1-D bulk copy
//     (TMA, cp.async.bulk) per K tile and per V tile into a ring of
//     shared-memory stages signalled by mbarriers; q of each (sequence, kv
//     head) unit comes the same way into a double-buffered slot.
//   * Four consumer warps: each owns B/4 rows of every block, computes the
//     scores of all G query heads of the GQA group with fp32 FMAs, keeps its
//     own running max / sum / output (online softmax) and accumulates P.V.
//     At the end of a unit the four states are merged through shared memory.
//   * Split units (a range boundary inside a unit): the CTA stores its
//     partial state (max, sum, unnormalised output) in the workspace and
//     bumps the unit's arrival counter; the last CTA to arrive merges all
//     partial states with the same rescaling rule and writes the output,
//     then resets the counter.  No second kernel, no host round trip.
//   * Masking: rows of the last block past seq_len get a score of -inf by
//     selection and are skipped in P.V, so whatever those rows hold (NaN
//     included) never reaches the result.
//   * Every wait is bounded (pa_device.cuh); a timeout raises the CTA's abort
//     flag, records PA_DEV_TIMEOUT, drains copies still in flight and returns.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "pa_decode_host.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

constexpr int kConsumerWarps = 4;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 32;  // + one producer warp
constexpr int kRingBytes = 64 * 1024;             // K+V bytes staged per CTA
constexpr int kMergeBarrier = 1;                  // named barrier of the consumer warps

template <int D, int B, int G>
struct Cfg {
  static constexpr int kTileElems = B * D;
  static constexpr int kTileBytes = kTileElems * 2;
  static constexpr int kStagesRaw = kRingBytes / (2 * kTileBytes);
  static constexpr int kStages = kStagesRaw > 16 ? 16 : kStagesRaw;
  static constexpr int TPW = B / kConsumerWarps;        // rows of a block per consumer warp
  static constexpr int LPT = (TPW >= 4) ? 8 : 32 / TPW;  // lanes sharing one row in q.k
  static constexpr int PT = 32 / LPT;                    // rows per q.k pass
  static constexpr int NPASS = TPW / PT;
  static constexpr int DPL = D / LPT;  // dims per lane in q.k
  static constexpr int VEC = DPL >= 8 ? 8 : DPL;
  static constexpr int NCHUNK = DPL / VEC;
  static constexpr int DPV = D / 32;                 // dims per lane in p.V
  static constexpr int kPartStride = G * (D + 2);    // floats per partial slot: m[G], l[G], acc[G][D]
  static_assert(B % kConsumerWarps == 0, "block size");
  static_assert(TPW % PT == 0, "rows per pass");
  static_assert(DPL % VEC == 0 && (VEC == 2 || VEC == 4 || VEC == 8), "q.k vector width");
  static_assert(DPV == 2 || DPV == 4, "p.V vector width");
};

template <int D, int B, int G>
struct __align__(128) DecodeSmem {
  using C = Cfg<D, B, G>;
  uint16_t k[C::kStages][C::kTileElems];
  uint16_t v[C::kStages][C::kTileElems];
  uint16_t q[2][G * D];
  float merge_acc[kConsumerWarps][G * D];
  float merge_m[kConsumerWarps][G];
  float merge_l[kConsumerWarps][G];
  float pbuf[kConsumerWarps][C::TPW][G];
  uint64_t full[C::kStages];
  uint64_t empty[C::kStages];
  uint64_t qfull[2];
  uint64_t qempty[2];
  RangeSmem range;
  int abort;
  int is_last;
  int issued;
  int consumed;
  int q_issued;
  int q_consumed;
};

template <bool kBf16, int D, int B, int G>
__global__ void __launch_bounds__(kThreads) pa_decode_kernel(const DecodeParams p) {
  using C = Cfg<D, B, G>;
  using Smem = DecodeSmem<D, B, G>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long cta = blockIdx.x;
  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;

  grid_dependency_wait();
  grid_launch_dependents();
  zero_empty_outputs<kThreads, B>(p, D);
  WorkRange wr;
  Cursor cur;
  if (!decode_prologue<kThreads, B, 1>(p, sm.range, wr, cur)) return;  // uniform across the CTA

  if (tid == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], kConsumerWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.qfull[i], 1);
      mbar_init(&sm.qempty[i], kConsumerWarps);
    }
    sm.abort = 0;
    sm.issued = 0;
    sm.consumed = 0;
    sm.q_issued = 0;
    sm.q_consumed = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const volatile int* abort_flag = &sm.abort;

  if (warp == kConsumerWarps) {
    // ===================== producer warp ======================================
    const uint64_t pol_stream = l2_policy_evict_first();
    int stage = 0, qslot = 0;
    uint32_t phase = 0, qphase = 0;
    int issued = 0, q_issued = 0;
    bool ok = true;
    if (p.test_flags & kFlagTestWithholdCopies) {
      // Test hook: issue nothing; the consumers' bounded waits must run out.
      if (lane == 0) {
        const uint64_t t0 = global_timer_ns();
        while (*abort_flag == 0 && global_timer_ns() - t0 < 4 * p.wait_limit_ns) {
        }
      }
      __syncwarp();
    } else {
      Seg sg;
      while (ok && next_seg<B, 1>(cur, sg, p)) {
        if (lane == 0) {
          ok = mbar_wait_bounded(&sm.qempty[qslot], qphase ^ 1u, abort_flag, p.wait_limit_ns);
          if (ok) {
            mbar_arrive_expect_tx(&sm.qfull[qslot], G * D * 2);
            const uint16_t* src = p.q + (static_cast<size_t>(sg.s) * Hq + static_cast<size_t>(sg.h) * G) * D;
            bulk_copy_g2s(sm.q[qslot], src, G * D * 2, &sm.qfull[qslot], pol_stream);
            ++q_issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        qslot ^= 1;
        if (qslot == 0) qphase ^= 1u;
        const int32_t* trow = p.block_tables + static_cast<size_t>(sg.s) * p.max_nb;
        for (int jb = sg.j0; jb < sg.j0 + sg.n && ok; jb += 32) {
          const int cnt = min(32, sg.j0 + sg.n - jb);
          int e = 0;
          if (lane < cnt) {
            e = __ldg(trow + jb + lane);
            if (e < 0 || e >= p.num_blocks) {
              record_status(p.status, PA_DEV_BAD_BLOCK_ID);
              e = 0;
            }
          }
          for (int k = 0; k < cnt; ++k) {
            const int phys = __shfl_sync(0xffffffffu, e, k);
            if (lane == 0) {
              ok = mbar_wait_bounded(&sm.empty[stage], phase ^ 1u, abort_flag, p.wait_limit_ns);
              if (ok) {
                const size_t tile = (static_cast<size_t>(phys) * Hkv + sg.h) * C::kTileElems;
                mbar_arrive_expect_tx(&sm.full[stage], 2 * C::kTileBytes);
                bulk_copy_g2s(sm.k[stage], p.k_pool + tile, C::kTileBytes, &sm.full[stage], pol_stream);
                bulk_copy_g2s(sm.v[stage], p.v_pool + tile, C::kTileBytes, &sm.full[stage], pol_stream);
                ++issued;
              }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    }
    if (lane == 0) {
      sm.issued = issued;
      sm.q_issued = q_issued;
      if (!ok) {
        sm.abort = 1;
        record_status(p.status, PA_DEV_TIMEOUT);
      }
    }
  } else {
    // ===================== consumer warps =====================================
    const int ctid = tid;  // 0..127
    const int c = lane % C::LPT;        // lane's column group inside its row
    const int rsub = lane / C::LPT;     // row inside a pass
    int stage = 0, qslot = 0;
    uint32_t phase = 0, qphase = 0;
    int consumed = 0, q_consumed = 0;
    bool ok = true;
    Seg sg;
    while (ok && next_seg<B, 1>(cur, sg, p)) {
      // ---- q of this unit, pre-multiplied by scale*log2(e)
      ok = mbar_wait_bounded(&sm.qfull[qslot], qphase, abort_flag, p.wait_limit_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      float qr[G][C::DPL];
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int k = 0; k < C::NCHUNK; ++k) {
          load_f32<kBf16, C::VEC>(&sm.q[qslot][g * D + (k * C::LPT + c) * C::VEC], &qr[g][k * C::VEC]);
        }
#pragma unroll
        for (int i = 0; i < C::DPL; ++i) qr[g][i] *= p.scale_log2;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.qempty[qslot]);
      ++q_consumed;
      qslot ^= 1;
      if (qslot == 0) qphase ^= 1u;

      float m[G], l[G], acc[G][C::DPV];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int i = 0; i < C::DPV; ++i) acc[g][i] = 0.f;
      }

      for (int i = 0; i < sg.n; ++i) {
        ok = mbar_wait_bounded(&sm.full[stage], phase, abort_flag, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const int j = sg.j0 + i;
        const int valid = (j == sg.nb - 1) ? sg.len - j * B : B;
        const uint16_t* Kt = sm.k[stage];
        const uint16_t* Vt = sm.v[stage];

        // ---- scores of this warp's rows for the G heads (log2 domain)
        float sc[C::NPASS][G];
#pragma unroll
        for (int ps = 0; ps < C::NPASS; ++ps) {
          const int r = warp * C::TPW + ps * C::PT + rsub;
          float dot[G];
#pragma unroll
          for (int g = 0; g < G; ++g) dot[g] = 0.f;
#pragma unroll
          for (int k = 0; k < C::NCHUNK; ++k) {
            float kf[C::VEC];
            load_f32<kBf16, C::VEC>(Kt + r * D + (k * C::LPT + c) * C::VEC, kf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
              for (int e = 0; e < C::VEC; ++e) dot[g] = fmaf(qr[g][k * C::VEC + e], kf[e], dot[g]);
            }
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int o = C::LPT / 2; o >= 1; o >>= 1) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], o);
            sc[ps][g] = (r < valid) ? dot[g] : -INFINITY;
          }
        }

        // ---- online softmax update (running max m, running sum l)
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float bm = sc[0][g];
#pragma unroll
          for (int ps = 1; ps < C::NPASS; ++ps) bm = fmaxf(bm, sc[ps][g]);
#pragma unroll
          for (int o = C::LPT; o < 32; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
          const float m_new = fmaxf(m[g], bm);
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          const float alpha = fast_exp2(m[g] - m_use);
          m[g] = m_new;
          float psum = 0.f;
#pragma unroll
          for (int ps = 0; ps < C::NPASS; ++ps) {
            const float pr = fast_exp2(sc[ps][g] - m_use);
            psum += pr;
            if (c == 0) sm.pbuf[warp][ps * C::PT + rsub][g] = pr;
          }
          l[g] = l[g] * alpha + psum;
#pragma unroll
          for (int e = 0; e < C::DPV; ++e) acc[g][e] *= alpha;
        }
        __syncwarp();

        // ---- P.V over this warp's valid rows
        int nv = valid - warp * C::TPW;
        nv = nv < 0 ? 0 : (nv > C::TPW ? C::TPW : nv);
#pragma unroll
        for (int t = 0; t < C::TPW; ++t) {
          if (t < nv) {
            const int r = warp * C::TPW + t;
            float vf[C::DPV];
            load_f32<kBf16, C::DPV>(Vt + r * D + lane * C::DPV, vf);
            float pt[G];
            if constexpr (G == 4) {
              const float4 pv = *reinterpret_cast<const float4*>(&sm.pbuf[warp][t][0]);
              pt[0] = pv.x;
              pt[1] = pv.y;
              pt[2] = pv.z;
              pt[3] = pv.w;
            } else {
#pragma unroll
              for (int g = 0; g < G; ++g) pt[g] = sm.pbuf[warp][t][g];
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
#pragma unroll
              for (int e = 0; e < C::DPV; ++e) acc[g][e] = fmaf(pt[g], vf[e], acc[g][e]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
        ++consumed;
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;

      // ---- merge the four warps' states of this segment
#pragma unroll
      for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int o = C::LPT; o < 32; o <<= 1) l[g] += __shfl_xor_sync(0xffffffffu, l[g], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          sm.merge_m[warp][g] = m[g];
          sm.merge_l[warp][g] = l[g];
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float* dst = &sm.merge_acc[warp][g * D + lane * C::DPV];
        if constexpr (C::DPV == 4) {
          *reinterpret_cast<float4*>(dst) = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
        } else {
          *reinterpret_cast<float2*>(dst) = make_float2(acc[g][0], acc[g][1]);
        }
      }
      named_barrier_sync(kMergeBarrier, kConsumerThreads);

      const bool whole_unit = (sg.j0 == sg.first && sg.j0 + sg.n == sg.nb);
      const long long F = sg.unit_first;
      float* my_part = nullptr;
      if (!whole_unit) {
        my_part = p.partials + partial_slot(cta, F, wr) * C::kPartStride;
      }
      uint16_t* out_row = p.out + (static_cast<size_t>(sg.s) * Hq + static_cast<size_t>(sg.h) * G) * D;
      for (int idx = ctid; idx < G * D / 2; idx += kConsumerThreads) {
        const int g = (2 * idx) / D, d = (2 * idx) % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.merge_m[w][g]);
        float L = 0.f, a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float sc_w = fast_exp2(sm.merge_m[w][g] - M);
          L = fmaf(sm.merge_l[w][g], sc_w, L);
          a0 = fmaf(sm.merge_acc[w][g * D + d], sc_w, a0);
          a1 = fmaf(sm.merge_acc[w][g * D + d + 1], sc_w, a1);
        }
        if (whole_unit) {
          const float inv = 1.f / L;
          *reinterpret_cast<uint32_t*>(out_row + g * D + d) = pack2<kBf16>(a0 * inv, a1 * inv);
        } else {
          if (d == 0) {
            my_part[g] = M;
            my_part[G + g] = L;
          }
          *reinterpret_cast<float2*>(&my_part[2 * G + g * D + d]) = make_float2(a0, a1);
        }
      }
      if (!whole_unit) {
        __threadfence();
        finish_split_unit<kBf16, D, G>(p, sg, wr, ctid, kConsumerThreads, &sm.is_last,
                                       [] { named_barrier_sync(kMergeBarrier, kConsumerThreads); });
      }
      named_barrier_sync(kMergeBarrier, kConsumerThreads);
    }
    if (tid == 0) {
      sm.consumed = consumed;
      sm.q_consumed = q_consumed;
    }
    if (!ok && lane == 0) {
      sm.abort = 1;
      record_status(p.status, PA_DEV_TIMEOUT);
    }
  }

  // ---- epilogue: after an abort, wait (bounded) for copies still in flight
  __syncthreads();
  if (tid == 0 && sm.abort) {
    for (int k = sm.consumed; k < sm.issued; ++k) {
      (void)mbar_wait_bounded(&sm.full[k % C::kStages], (k / C::kStages) & 1, nullptr, p.wait_limit_ns);
    }
    for (int k = sm.q_consumed; k < sm.q_issued; ++k) {
      (void)mbar_wait_bounded(&sm.qfull[k & 1], (k >> 1) & 1, nullptr, p.wait_limit_ns);
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <bool kBf16, int D, int B, int G>
static cudaError_t launch_cuda_cores(const Variant& v, const DecodeParams& prm, int ctas, cudaStream_t stream) {
  return launch_overlapped(pa_decode_kernel<kBf16, D, B, G>, dim3(ctas), dim3(kThreads),
                           static_cast<size_t>(v.smem_bytes), stream, prm);
}

template <bool kBf16, int D, int B, int G>
Variant make_variant() {
  return Variant{reinterpret_cast<const void*>(&pa_decode_kernel<kBf16, D, B, G>), kThreads,
                 static_cast<int>(sizeof(DecodeSmem<D, B, G>)), Cfg<D, B, G>::kPartStride,
                 &launch_cuda_cores<kBf16, D, B, G>, 0};
}

template <bool kBf16, int D, int B>
bool pick_g(int G, Variant& v) {
  switch (G) {
    case 1: v = make_variant<kBf16, D, B, 1>(); return true;
    case 2: v = make_variant<kBf16, D, B, 2>(); return true;
    case 4: v = make_variant<kBf16, D, B, 4>(); return true;
    case 8: v = make_variant<kBf16, D, B, 8>(); return true;
    default: return false;
  }
}

template <bool kBf16, int D>
bool pick_b(int B, int G, Variant& v) {
  switch (B) {
    case 8: return pick_g<kBf16, D, 8>(G, v);
    case 16: return pick_g<kBf16, D, 16>(G, v);
    case 32: return pick_g<kBf16, D, 32>(G, v);
    default: return false;
  }
}

template <bool kBf16>
bool pick_d(int D, int B, int G, Variant& v) {
  switch (D) {
    case 64: return pick_b<kBf16, 64>(B, G, v);
    case 128: return pick_b<kBf16, 128>(B, G, v);
    default: return false;
  }
}

// The tensor-core kernel where one applies (unless the caller asks for CUDA
// cores only), else the CUDA-core kernel.
static bool select_variant(const pa_pool_desc& pool, int num_q_heads, int flags, Variant& v) {
  if (pool.num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % pool.num_kv_heads != 0) return false;
  const int G = num_q_heads / pool.num_kv_heads;
  if ((flags & PA_DECODE_CUDA_CORES_ONLY) == 0 && select_tc_variant(pool, G, v)) return true;
  if (pool.dtype == PA_BF16) return pick_d<true>(pool.head_dim, pool.block_size, G, v);
  if (pool.dtype == PA_FP16) return pick_d<false>(pool.head_dim, pool.block_size, G, v);
  return false;
}

// Resident CTAs per SM times the SM count for a variant on the current
// device; also raises the kernel's dynamic shared memory limit.  Cached per
// device and kernel.
static bool grid_size_for(const Variant& v, int& ctas) {
  struct Entry {
    int device;
    const void* fn;
    int ctas;
  };
  static std::mutex mu;
  static Entry cache[512];
  static int n_cache = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_cache; ++i) {
      if (cache[i].device == dev && cache[i].fn == v.kernel) {
        ctas = cache[i].ctas;
        return true;
      }
    }
  }
  if (cudaFuncSetAttribute(v.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, v.smem_bytes) != cudaSuccess)
    return false;
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v.kernel, v.threads, v.smem_bytes) != cudaSuccess)
    return false;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
  if (per_sm < 1) return false;
  ctas = per_sm * sms;
  std::lock_guard<std::mutex> lock(mu);
  if (n_cache < 512) cache[n_cache++] = Entry{dev, v.kernel, ctas};
  return true;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static size_t partials_bytes(int ctas, int part_stride) {
  return align_up(static_cast<size_t>(ctas) * 2 * part_stride * sizeof(float), 256);
}

// [partial states][grid barrier words][arrival counters]
static size_t workspace_bytes_for(int num_seqs, int num_kv_heads, int ctas, int part_stride) {
  const size_t counters = align_up(static_cast<size_t>(num_seqs) * num_kv_heads * sizeof(int32_t), 256);
  return partials_bytes(ctas, part_stride) + kGridSyncBytes + counters;
}

static bool pool_shape_ok(const pa_pool_desc* pool) {
  return pool != nullptr && pool->num_blocks > 0 && pool->block_size > 0 && pool->num_kv_heads > 0 &&
         pool->head_dim > 0 && (pool->dtype == PA_FP16 || pool->dtype == PA_BF16);
}

// CTA count: an explicit request, else the resident maximum.  Either way the
// kernel's shared-memory attribute is set.
static int resolve_ctas(const Variant& v, const pa_decode_opts* opts) {
  int ctas = 0;
  if (!grid_size_for(v, ctas)) return 0;
  if (opts != nullptr && opts->num_ctas > 0) return opts->num_ctas;
  return ctas;
}

static int opts_flags(const pa_decode_opts* opts) { return opts != nullptr ? opts->flags : 0; }

constexpr int kKnownFlags =
    PA_DECODE_TEST_WITHHOLD_COPIES | PA_DECODE_CUDA_CORES_ONLY | PA_DECODE_TEST_SKIP_UPDATE_ARRIVAL;

// Shared argument checks of the decode entry points.
static pa_status check_decode_args(const void* q, const void* k_pool, const void* v_pool,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                   int32_t num_seqs, int32_t num_q_heads, float scale, const void* out,
                                   const pa_pool_desc* pool) {
  if (!pool_shape_ok(pool) || num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0) {
    return PA_ERR_INVALID_ARG;
  }
  if (num_seqs == 0) return PA_OK;
  if (q == nullptr || k_pool == nullptr || v_pool == nullptr || block_tables == nullptr || seq_lens == nullptr ||
      out == nullptr) {
    return PA_ERR_INVALID_ARG;
  }
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out) || !std::isfinite(scale)) {
    return PA_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(max_blocks_per_seq) * pool->block_size > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

static DecodeParams make_params(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                                int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs,
                                int32_t num_q_heads, float scale, void* out, void* scratch, int ctas,
                                int part_stride, int32_t* dev_status, const pa_pool_desc* pool, int flags) {
  DecodeParams prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.k_pool = static_cast<const uint16_t*>(k_pool);
  prm.v_pool = static_cast<const uint16_t*>(v_pool);
  prm.block_tables = block_tables;
  prm.seq_lens = seq_lens;
  prm.out = static_cast<uint16_t*>(out);
  prm.partials = static_cast<float*>(scratch);
  prm.grid_sync = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + partials_bytes(ctas, part_stride));
  prm.counters = prm.grid_sync + kGridSyncBytes / sizeof(int32_t);
  prm.status = dev_status;
  prm.max_nb = max_blocks_per_seq;
  prm.num_seqs = num_seqs;
  prm.num_q_heads = num_q_heads;
  prm.num_kv_heads = pool->num_kv_heads;
  prm.num_blocks = pool->num_blocks;
  prm.scale_log2 = scale * 1.4426950408889634f;
  const int test_flags = flags & (PA_DECODE_TEST_WITHHOLD_COPIES | PA_DECODE_TEST_SKIP_UPDATE_ARRIVAL);
  prm.wait_limit_ns = test_flags != 0 ? 20ull * 1000 * 1000 : 2ull * 1000 * 1000 * 1000;
  prm.test_flags = test_flags;
  prm.q_len = 1;
  prm.q_tiles = 1;
  prm.group_starts = nullptr;
  prm.group_prefix = nullptr;
  prm.num_groups = 0;
  prm.unit_cost = 0;
  prm.lse = nullptr;
  prm.upd_k = nullptr;
  prm.upd_v = nullptr;
  prm.upd_slots = nullptr;
  prm.upd_num_tokens = 0;
  return prm;
}

// ---- cache update ahead of a decode (pa_decode_update and friends) -----------

static bool has_update(const pa_cache_update* u) {
  return u != nullptr && (u->num_copy_pairs > 0 || u->num_tokens > 0);
}

static bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// Host-visible checks of an update (NULL is no update).
static bool update_args_ok(const pa_cache_update* u) {
  if (u == nullptr) return true;
  if (u->num_copy_pairs < 0 || u->num_tokens < 0) return false;
  if (u->num_copy_pairs > 0 && (u->copy_pairs == nullptr || !aligned8(u->copy_pairs))) return false;
  if (u->num_tokens > 0 && (u->k == nullptr || u->v == nullptr || u->slot_mapping == nullptr ||
                            !aligned16(u->k) || !aligned16(u->v) || !aligned8(u->slot_mapping))) {
    return false;
  }
  return true;
}

// The update as its own two kernels, enqueued before the decode.
static pa_status enqueue_update(const pa_cache_update* u, void* k_pool, void* v_pool, int32_t* dev_status,
                                const pa_pool_desc* pool, void* stream) {
  if (!has_update(u)) return PA_OK;
  pa_status st = PA_OK;
  if (u->num_copy_pairs > 0) st = pa_copy_blocks(u->copy_pairs, u->num_copy_pairs, k_pool, v_pool, dev_status, pool, stream);
  if (st == PA_OK && u->num_tokens > 0) {
    st = pa_cache_write(u->k, u->v, u->slot_mapping, u->num_tokens, k_pool, v_pool, dev_status, pool, stream);
  }
  return st;
}

// Launch a decode variant after the update.  The block copies run as their
// own kernel ahead of it (inside the decode launch they measured slower:
// one CTA per SM keeps fewer copies in flight, and their barrier delayed
// every CTA's first load).  The new tokens' stores run inside the launch
// where the variant takes them and the whole grid can be resident at once
// (its grid-wide barrier needs every CTA on an SM), else as pa_cache_write.
static pa_status launch_decode(const Variant& v, DecodeParams& prm, int ctas, const pa_cache_update* u,
                               void* k_pool, void* v_pool, const pa_pool_desc* pool, void* stream) {
  if (has_update(u)) {
    int resident = 0;
    if (v.fuses_update && grid_size_for(v, resident) && ctas <= resident) {
      if (u->num_copy_pairs > 0) {
        const pa_status st =
            pa_copy_blocks(u->copy_pairs, u->num_copy_pairs, k_pool, v_pool, prm.status, pool, stream);
        if (st != PA_OK) return st;
      }
      if (u->num_tokens > 0) {
        prm.upd_k = static_cast<const uint4*>(u->k);
        prm.upd_v = static_cast<const uint4*>(u->v);
        prm.upd_slots = u->slot_mapping;
        prm.upd_num_tokens = u->num_tokens;
      }
    } else {
      const pa_status st = enqueue_update(u, k_pool, v_pool, prm.status, pool, stream);
      if (st != PA_OK) return st;
    }
  }
  return v.launch(v, prm, ctas, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// CTA count for a workspace-size query: an explicit request needs no device.
static bool query_ctas(const Variant& v, const pa_decode_opts* opts, int& ctas) {
  if (opts != nullptr && opts->num_ctas > 0) {
    ctas = opts->num_ctas;
    return true;
  }
  return grid_size_for(v, ctas);
}

static bool group_of(const pa_pool_desc& pool, int num_q_heads, int& G) {
  if (pool.num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % pool.num_kv_heads != 0) return false;
  G = num_q_heads / pool.num_kv_heads;
  return true;
}

static bool opts_ok(const pa_decode_opts* opts) {
  return opts == nullptr || (opts->num_ctas >= 0 && (opts->flags & ~kKnownFlags) == 0);
}

// ---- multi-query decode ------------------------------------------------------

// The variant and its row tiles (units) per sequence; false also when the
// units of the batch overflow the unit index.
static bool multi_variant(const pa_pool_desc& pool, int num_seqs, int num_q_heads, int q_len, Variant& v,
                          int& tiles) {
  int G = 0;
  if (!group_of(pool, num_q_heads, G) || !select_tc_multi_variant(pool, G, q_len, v, tiles)) return false;
  return tiles >= 1 && static_cast<long long>(num_seqs) * tiles <= 0x7fffffffLL;
}

// ---- shared-prefix decode ----------------------------------------------------
// One launch over (group, kv head) units; the workspace is a decode
// workspace sized for the group variant's rows (counters per group fit in the
// per-sequence counter array since there are no more groups than sequences).

static bool group_variant(const pa_pool_desc& pool, int num_q_heads, int max_group_size, Variant& v) {
  int G = 0;
  return max_group_size >= 1 && group_of(pool, num_q_heads, G) && select_tc_group_variant(pool, G, max_group_size, v);
}

}  // namespace pa

using namespace pa;

extern "C" size_t pa_decode_workspace_bytes_ex(int32_t num_seqs, int32_t num_q_heads, const pa_pool_desc* pool,
                                               const pa_decode_opts* opts) {
  if (num_seqs < 0 || !pool_shape_ok(pool)) return 0;
  Variant v;
  if (!select_variant(*pool, num_q_heads, opts_flags(opts), v)) return 0;
  int ctas = 0;
  if (opts != nullptr && opts->num_ctas > 0) {
    ctas = opts->num_ctas;  // no device query needed
  } else if (!grid_size_for(v, ctas)) {
    return 0;
  }
  return workspace_bytes_for(num_seqs, pool->num_kv_heads, ctas, v.part_stride);
}

extern "C" size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, const pa_pool_desc* pool) {
  return pa_decode_workspace_bytes_ex(num_seqs, num_q_heads, pool, nullptr);
}

static pa_status decode_impl(const pa_cache_update* upd, const void* q, const void* k_pool, const void* v_pool,
                             const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                             int32_t num_seqs, int32_t num_q_heads, float scale, void* out, void* workspace,
                             size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                             const pa_decode_opts* opts, void* stream, float* lse = nullptr) {
  pa_status st = check_decode_args(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                    num_q_heads, scale, out, pool);
  if (st != PA_OK) return st;
  if (!update_args_ok(upd)) return PA_ERR_INVALID_ARG;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return enqueue_update(upd, const_cast<void*>(k_pool), const_cast<void*>(v_pool), dev_status, pool, stream);
  if (opts != nullptr && (opts->num_ctas < 0 || (opts->flags & ~kKnownFlags) != 0)) return PA_ERR_INVALID_ARG;
  Variant v;
  if (!select_variant(*pool, num_q_heads, opts_flags(opts), v)) return PA_ERR_UNSUPPORTED;
  const int ctas = resolve_ctas(v, opts);
  if (ctas <= 0) return PA_ERR_CUDA;
  const size_t need = workspace_bytes_for(num_seqs, pool->num_kv_heads, ctas, v.part_stride);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;
  DecodeParams prm = make_params(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                       num_q_heads, scale, out, workspace, ctas, v.part_stride, dev_status, pool,
                                       opts_flags(opts));
  prm.unit_cost = v.unit_cost;
  if (lse != nullptr) {
    if (!v.fuses_update) return PA_ERR_UNSUPPORTED;  // the log normalisers come from the tensor-core kernel
    prm.lse = lse;
  }
  return launch_decode(v, prm, ctas, upd, const_cast<void*>(k_pool), const_cast<void*>(v_pool), pool, stream);
}

extern "C" pa_status pa_decode_lse(const void* q, const void* k_pool, const void* v_pool,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                   int32_t num_seqs, int32_t num_q_heads, float scale, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                   const pa_pool_desc* pool, const pa_decode_opts* opts, void* stream) {
  if (lse == nullptr && num_seqs > 0) return PA_ERR_INVALID_ARG;
  return decode_impl(nullptr, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                     scale, out, workspace, workspace_bytes, dev_status, pool, opts, stream, lse);
}

extern "C" pa_status pa_decode_ex(const void* q, const void* k_pool, const void* v_pool,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                  int32_t num_seqs, int32_t num_q_heads, float scale, void* out, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                                  const pa_decode_opts* opts, void* stream) {
  return decode_impl(nullptr, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                     scale, out, workspace, workspace_bytes, dev_status, pool, opts, stream);
}

extern "C" pa_status pa_decode_update(const pa_cache_update* update, const void* q, void* k_pool, void* v_pool,
                                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
                                      void* out, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                      const pa_pool_desc* pool, const pa_decode_opts* opts, void* stream) {
  return decode_impl(update, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                     scale, out, workspace, workspace_bytes, dev_status, pool, opts, stream);
}

extern "C" pa_status pa_decode(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables,
                               int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs,
                               int32_t num_q_heads, float scale, void* out, void* workspace,
                               size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                               void* stream) {
  return pa_decode_ex(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads, scale,
                      out, workspace, workspace_bytes, dev_status, pool, nullptr, stream);
}

extern "C" size_t pa_decode_multi_workspace_bytes(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                                  const pa_pool_desc* pool, const pa_decode_opts* opts) {
  if (q_len == 1) return pa_decode_workspace_bytes_ex(num_seqs, num_q_heads, pool, opts);
  if (num_seqs < 0 || q_len < 1 || !pool_shape_ok(pool)) return 0;
  Variant v;
  int ctas = 0, tiles = 0;
  if (!multi_variant(*pool, num_seqs, num_q_heads, q_len, v, tiles) || !query_ctas(v, opts, ctas)) return 0;
  return workspace_bytes_for(num_seqs * tiles, pool->num_kv_heads, ctas, v.part_stride);
}

static pa_status multi_impl(const pa_cache_update* upd, const void* q, const void* k_pool, const void* v_pool,
                            const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                            int32_t num_seqs, int32_t q_len, int32_t num_q_heads, float scale, void* out,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                            const pa_decode_opts* opts, void* stream) {
  if (q_len < 1) return PA_ERR_INVALID_ARG;
  if (q_len == 1) {
    return decode_impl(upd, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                       scale, out, workspace, workspace_bytes, dev_status, pool, opts, stream);
  }
  pa_status st = check_decode_args(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                    num_q_heads, scale, out, pool);
  if (st != PA_OK) return st;
  if (!update_args_ok(upd)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return enqueue_update(upd, const_cast<void*>(k_pool), const_cast<void*>(v_pool), dev_status, pool, stream);
  if (!opts_ok(opts)) return PA_ERR_INVALID_ARG;
  if (static_cast<long long>(num_seqs) * q_len > 0x7fffffffLL) return PA_ERR_INVALID_ARG;
  if ((opts_flags(opts) & PA_DECODE_CUDA_CORES_ONLY) != 0) return PA_ERR_UNSUPPORTED;
  Variant v;
  int tiles = 0;
  if (!multi_variant(*pool, num_seqs, num_q_heads, q_len, v, tiles)) return PA_ERR_UNSUPPORTED;
  const int ctas = resolve_ctas(v, opts);
  if (ctas <= 0) return PA_ERR_CUDA;
  const size_t need = workspace_bytes_for(num_seqs * tiles, pool->num_kv_heads, ctas, v.part_stride);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;
  DecodeParams prm = make_params(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                 num_q_heads, scale, out, workspace, ctas, v.part_stride, dev_status, pool,
                                 opts_flags(opts));
  prm.q_len = q_len;
  prm.q_tiles = tiles;
  prm.unit_cost = v.unit_cost;
  return launch_decode(v, prm, ctas, upd, const_cast<void*>(k_pool), const_cast<void*>(v_pool), pool, stream);
}

extern "C" pa_status pa_decode_multi(const void* q, const void* k_pool, const void* v_pool,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* seq_lens, int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                     float scale, void* out, void* workspace, size_t workspace_bytes,
                                     int32_t* dev_status, const pa_pool_desc* pool, const pa_decode_opts* opts,
                                     void* stream) {
  return multi_impl(nullptr, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, q_len,
                    num_q_heads, scale, out, workspace, workspace_bytes, dev_status, pool, opts, stream);
}

extern "C" pa_status pa_decode_multi_update(const pa_cache_update* update, const void* q, void* k_pool,
                                            void* v_pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                            const int32_t* seq_lens, int32_t num_seqs, int32_t q_len,
                                            int32_t num_q_heads, float scale, void* out, void* workspace,
                                            size_t workspace_bytes, int32_t* dev_status, const pa_pool_desc* pool,
                                            const pa_decode_opts* opts, void* stream) {
  return multi_impl(update, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs, q_len,
                    num_q_heads, scale, out, workspace, workspace_bytes, dev_status, pool, opts, stream);
}

extern "C" size_t pa_decode_shared_prefix_workspace_bytes(int32_t num_seqs, int32_t max_group_size,
                                                          int32_t num_q_heads, const pa_pool_desc* pool,
                                                          const pa_decode_opts* opts) {
  if (num_seqs < 0 || !pool_shape_ok(pool)) return 0;
  Variant v;
  int ctas = 0;
  if (!group_variant(*pool, num_q_heads, max_group_size, v) || !query_ctas(v, opts, ctas)) return 0;
  return workspace_bytes_for(num_seqs, pool->num_kv_heads, ctas, v.part_stride);
}

static pa_status shared_prefix_impl(const pa_cache_update* upd, const void* q, const void* k_pool,
                                    const void* v_pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
                                    const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                                    const int32_t* group_starts, const int32_t* group_prefix_blocks,
                                    int32_t num_groups, int32_t max_group_size, float scale, void* out,
                                    void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                    const pa_pool_desc* pool, const pa_decode_opts* opts, void* stream) {
  pa_status st = check_decode_args(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                    num_q_heads, scale, out, pool);
  if (st != PA_OK) return st;
  if (num_groups < 0 || max_group_size < 1 || (num_seqs > 0 && num_groups == 0) || num_groups > num_seqs) {
    return PA_ERR_INVALID_ARG;
  }
  if (!update_args_ok(upd)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return enqueue_update(upd, const_cast<void*>(k_pool), const_cast<void*>(v_pool), dev_status, pool, stream);
  if (group_starts == nullptr || group_prefix_blocks == nullptr) return PA_ERR_INVALID_ARG;
  if (!opts_ok(opts)) return PA_ERR_INVALID_ARG;
  if ((opts_flags(opts) & PA_DECODE_CUDA_CORES_ONLY) != 0) return PA_ERR_UNSUPPORTED;
  Variant v;
  if (!group_variant(*pool, num_q_heads, max_group_size, v)) return PA_ERR_UNSUPPORTED;
  const int ctas = resolve_ctas(v, opts);
  if (ctas <= 0) return PA_ERR_CUDA;
  const size_t need = workspace_bytes_for(num_seqs, pool->num_kv_heads, ctas, v.part_stride);
  if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)) return PA_ERR_WORKSPACE;
  DecodeParams prm = make_params(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                 num_q_heads, scale, out, workspace, ctas, v.part_stride, dev_status, pool,
                                 opts_flags(opts));
  prm.group_starts = group_starts;
  prm.group_prefix = group_prefix_blocks;
  prm.num_groups = num_groups;
  prm.unit_cost = v.unit_cost;
  return launch_decode(v, prm, ctas, upd, const_cast<void*>(k_pool), const_cast<void*>(v_pool), pool, stream);
}

extern "C" pa_status pa_decode_shared_prefix(const void* q, const void* k_pool, const void* v_pool,
                                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                                             const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                                             const int32_t* group_starts, const int32_t* group_prefix_blocks,
                                             int32_t num_groups, int32_t max_group_size, float scale, void* out,
                                             void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                             const pa_pool_desc* pool, const pa_decode_opts* opts, void* stream) {
  return shared_prefix_impl(nullptr, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                            num_q_heads, group_starts, group_prefix_blocks, num_groups, max_group_size, scale, out,
                            workspace, workspace_bytes, dev_status, pool, opts, stream);
}

extern "C" pa_status pa_decode_shared_prefix_update(const pa_cache_update* update, const void* q, void* k_pool,
                                                    void* v_pool, const int32_t* block_tables,
                                                    int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                                    int32_t num_seqs, int32_t num_q_heads,
                                                    const int32_t* group_starts, const int32_t* group_prefix_blocks,
                                                    int32_t num_groups, int32_t max_group_size, float scale,
                                                    void* out, void* workspace, size_t workspace_bytes,
                                                    int32_t* dev_status, const pa_pool_desc* pool,
                                                    const pa_decode_opts* opts, void* stream) {
  return shared_prefix_impl(update, q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                            num_q_heads, group_starts, group_prefix_blocks, num_groups, max_group_size, scale, out,
                            workspace, workspace_bytes, dev_status, pool, opts, stream);
}

// ---------------------------------------------------------------------------
// pa_decode_no_alloc: the same decode with its scratch (partial states and
// arrival counters) in a fixed array of libpa's own device memory, for
// callers that cannot allocate device memory themselves.
// ---------------------------------------------------------------------------

namespace pa {

constexpr size_t kNoAllocScratchBytes = PA_DECODE_NO_ALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Held by every GPU that loads libpa, until the process exits.  Host code must
// not pass this name to a kernel: on the host it is only a stand-in for the
// symbol, so its device address is looked up below.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// The current context's process-unique id (cuCtxGetId never hands out an id
// twice in a process), or 0 when no context is current or the driver entry
// points are missing.  Reached through the runtime's driver entry point
// table, so libpa needs no link against the driver library.
static unsigned long long current_context_id() {
  using GetCurrentFn = int (*)(void**);
  using GetIdFn = int (*)(void*, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrentFn>(f);
    }
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess) {
      get_id = reinterpret_cast<GetIdFn>(f);
    }
    looked_up = true;
  }
  void* ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != 0 || ctx == nullptr) return 0;
  return get_id(ctx, &id) == 0 ? id : 0;
}

// Device address of g_decode_scratch on the current device.  It is looked up
// with that device current on the first call, and again whenever the
// device's current context is another one than at the last lookup (after a
// cudaDeviceReset the module is loaded anew and the array may sit
// elsewhere); otherwise the cached address is used.
static bool no_alloc_scratch_address(void** addr) {
  static std::mutex mu;
  static void* cached[kMaxDevices] = {};
  static unsigned long long cached_ctx[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (cached[dev] == nullptr || ctx == 0 || ctx != cached_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return false;
    cached[dev] = p;
    // the lookup makes the device's primary context current if none was
    cached_ctx[dev] = current_context_id();
  }
  *addr = cached[dev];
  return true;
}

}  // namespace pa

extern "C" pa_status pa_decode_no_alloc(const void* q, const void* k_pool, const void* v_pool,
                                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                                        const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
                                        void* out, int32_t* dev_status, const pa_pool_desc* pool, void* stream) {
  pa_status st = check_decode_args(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                    num_q_heads, scale, out, pool);
  if (st != PA_OK || num_seqs == 0) return st;
  Variant v;
  if (!select_variant(*pool, num_q_heads, 0, v)) return PA_ERR_UNSUPPORTED;
  const int ctas = resolve_ctas(v, nullptr);
  if (ctas <= 0) return PA_ERR_CUDA;
  if (workspace_bytes_for(num_seqs, pool->num_kv_heads, ctas, v.part_stride) > kNoAllocScratchBytes) {
    return PA_ERR_SCRATCH_LIMIT;
  }
  void* scratch = nullptr;
  if (!no_alloc_scratch_address(&scratch)) return PA_ERR_CUDA;
  DecodeParams prm = make_params(q, k_pool, v_pool, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                       num_q_heads, scale, out, scratch, ctas, v.part_stride, dev_status, pool, 0);
  // The array keeps whatever the previous call left; the arrival counters
  // must start at zero, so clear them on the caller's stream first.
  if (cudaMemsetAsync(prm.counters, 0, static_cast<size_t>(num_seqs) * pool->num_kv_heads * sizeof(int32_t),
                      static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    return PA_ERR_CUDA;
  }
  prm.unit_cost = v.unit_cost;
  return v.launch(v, prm, ctas, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
