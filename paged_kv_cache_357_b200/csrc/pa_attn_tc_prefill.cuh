// Multi-query paged attention in query-major tiles (prefill chunks and long
// speculative runs) on tensor cores, sm_100a.  Each sequence brings q_len
// new query positions; position i sees the sequence's tokens up to
// seq_len - q_len + i (CSDN "PagedAttention：分页注意力", §"2026年最新进展"
// items 1-2), merged over the paged blocks by the online softmax (study
// notes ch.05 §4; vLLM blog §"关键细节" 2).
//
// A unit is 128 query rows: the G heads of one kv head at 128 / G
// consecutive positions of one sequence (row r = position offset r / G,
// head r % G).  Per 128-token chunk of the sequence's blocks:
//
//   S[row, token] = Q[row, :] . K_chunk[token, :]        (M=128, N=128, K=128)
//   O[row, d]    += P[row, token] . V_chunk[token, d]     (M=128, N=128, K=16 a step)
//
// The rows sit in TMEM lanes, so a softmax thread owns (half of) row r of
// every chunk: its causal limit, running sum and rescale are its own; only
// a chunk's max passes between the two threads that share a row.  P enters
// PV as a 16-bit head and a 16-bit residual (two MMAs a step), as in the
// decode kernel.  Against the decode's token-major tile (128 tokens x at most 32
// rows, pa_attn_tc.cuh) a tile does four times the arithmetic per MMA and
// per loaded K/V chunk.
//
// Roles (384 threads, one CTA per SM): warp 0 loads q and K (TMA, 128-byte
// swizzle), warp 1 issues QK, warp 2 loads V, warp 3 issues PV, warps 4-11
// run the softmax: two warpgroups, each row split between them by tokens
// (and O by head_dim columns).  Work partition, bounded waits and
// the split-unit merge (by the CTA holding a unit's first piece) follow
// pa_attn_tc.cuh and pa_decode_common.cuh; so does the geometry of a chunk's
// blocks (Blk<B>: blocks of 8, 16 or 32 tokens).
#pragma once

#include "pa_attn_tc.cuh"

namespace pa {
namespace tc {
namespace pf {

constexpr int kRows = 128;                        // query rows of a unit: MMA M
constexpr int kChunk = 128;                       // tokens per chunk: MMA N of QK
constexpr int kKStages = 2, kVStages = 2;
constexpr int kQHalf = kRows * kRowBytes;         // 16 KB: head_dim [0, 64) (or [64, 128)) of the 128 rows
constexpr int kQBytes = 2 * kQHalf;
constexpr int kKHalf = kChunk * kRowBytes;        // 16 KB: one head_dim half of a chunk's tokens
constexpr int kStageBytes = 2 * kKHalf;           // 32 KB: one chunk of K or V
constexpr int kHalfChunk = kChunk / 2;            // tokens of a chunk per softmax warpgroup
constexpr int kThreads = 384;                     // control warpgroup + two softmax warpgroups
// The control warpgroup hands registers to the softmax warpgroups
// (setmaxnreg) inside the launch's 168 a thread: 128 x 80 + 256 x 208.
constexpr int kCtrlRegs = 80, kSoftmaxRegs = 208, kLaunchRegs = 168;
static_assert(128 * kCtrlRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kPairBarrier = 1;                   // named barrier of the two softmax warpgroups
// TMEM: kSBufs S buffers of 128 columns (P written over S once read), then
// kOBufs O accumulators of 128 columns.  Three S buffers let QK run a chunk
// further ahead of the softmax than two; one O buffer then makes a unit's
// first PV wait for the previous unit's finish.
constexpr int kSBufs = 3, kOBufs = 1;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = kSBufs * kChunk;
constexpr uint32_t kTmemCols = 512;
static_assert(kColO + kOBufs * D <= kTmemCols, "S and O buffers fit the 512 TMEM columns");
constexpr int kPartStride = kRows * (D + 2);      // floats per partial slot: m, l, acc per row

static_assert(kChunk == kChunkTok, "a chunk has the decode kernel's block geometry (Blk<B>)");

struct Smem {
  uint8_t kbuf[kKStages][kStageBytes];  // 1024-aligned regions
  uint8_t vbuf[kVStages][kStageBytes];
  uint8_t q[2][kQBytes];                // [half][128 rows][64]
  uint64_t kfull[kKStages];
  uint64_t kempty[kKStages];
  uint64_t vfull[kVStages];
  uint64_t vempty[kVStages];
  uint64_t qfull[2];
  uint64_t qempty[2];
  // per S buffer (chunk c uses buffer c % kSBufs): S written by QK, P
  // written over it by the softmax, and the chunk's PV complete (which frees
  // the buffer for QK of chunk c + kSBufs).  No waiter can fall two phases
  // behind.
  uint64_t s_full[kSBufs];
  uint64_t p_full[kSBufs];
  uint64_t pv_done[kSBufs];
  uint64_t unit_done[kOBufs];           // per O buffer: every PV of its unit has completed
  uint64_t o_free[kOBufs];              // a unit's O buffer has been read by its finish
  uint64_t mma_done[2];
  alignas(16) float red[2][2][kRows];   // per chunk parity and warpgroup: each row's max over its tokens
  alignas(16) float lsum[2][kRows];     // per warpgroup: a finished unit's row sums
  RangeSmem range;
  uint32_t tmem_base;
  int abort;
  int merge_ok;
  int k_issued, k_consumed, v_issued, v_consumed, q_issued, q_consumed;
};

constexpr int smem_bytes() { return static_cast<int>(sizeof(Smem)) + 1024; }
static_assert(smem_bytes() <= kMaxSmemPerCta, "shared memory of one CTA");

// Packed fp32 pairs: sm_100's two-lane FFMA, FADD, FSUB and FMUL each do
// two independent IEEE single-precision operations (round to nearest, no
// flush) in one instruction; the three-input max takes two new values a step.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n"
      "  .reg .b64 ra, rb, rc, rd;\n"
      "  mov.b64 ra, {%2, %3};\n"
      "  mov.b64 rb, {%4, %5};\n"
      "  mov.b64 rc, {%6, %7};\n"
      "  fma.rn.f32x2 rd, ra, rb, rc;\n"
      "  mov.b64 {%0, %1}, rd;\n"
      "}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

#define PA_PF_BINARY_F32X2(name, op)                                          \
  __device__ __forceinline__ float2 name(float2 a, float2 b) {                \
    float2 d;                                                                 \
    asm("{\n"                                                                 \
        "  .reg .b64 ra, rb, rd;\n"                                           \
        "  mov.b64 ra, {%2, %3};\n"                                           \
        "  mov.b64 rb, {%4, %5};\n"                                           \
        "  " op ".rn.f32x2 rd, ra, rb;\n"                                     \
        "  mov.b64 {%0, %1}, rd;\n"                                           \
        "}\n"                                                                 \
        : "=f"(d.x), "=f"(d.y)                                                \
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));                            \
    return d;                                                                 \
  }
PA_PF_BINARY_F32X2(add2, "add")
PA_PF_BINARY_F32X2(sub2, "sub")
PA_PF_BINARY_F32X2(mul2, "mul")
#undef PA_PF_BINARY_F32X2

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two probabilities as a 16-bit head pair and a 16-bit residual pair (P =
// head + residual, about 15 significant bits).  bf16 takes the upper half
// of each fp32 word (truncation: the head then leaves an exact fp32
// remainder, whose own upper half is the residual), with byte permutes and
// masks on the integer pipe, not conversions; fp16 rounds with the
// conversion instruction.
template <bool kBf16>
__device__ __forceinline__ void split_pair(float a0, float a1, uint32_t& head, uint32_t& resid) {
  if constexpr (kBf16) {
    const uint32_t u0 = __float_as_uint(a0), u1 = __float_as_uint(a1);
    head = __byte_perm(u0, u1, 0x7632);
    const float2 r = sub2(make_float2(a0, a1),
                          make_float2(__uint_as_float(u0 & 0xffff0000u), __uint_as_float(u1 & 0xffff0000u)));
    resid = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
  } else {
    head = pack2<false>(a0, a1);
    float h0, h1;
    unpack2<false>(head, h0, h1);
    resid = pack2<false>(a0 - h0, a1 - h1);
  }
}

// D[tmem] (+)= A[tmem] . B[smem desc], kind::f16, fp32 accumulate: A is
// M=128 lanes by K=16 16-bit values, two to a 32-bit column (the lower
// half holding the even K index).
__device__ __forceinline__ void umma_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  setp.ne.b32 p, %4, 0;\n"
      "  tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      "}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The chunks of one segment (a tile's blocks [j0, j0 + n) of its sequence).
template <int RG, int B>
struct Walk {
  static constexpr int CB = Blk<B>::CB;
  int seq, j, jend, len, pos0;
  __device__ __forceinline__ void start(const DecodeParams& p, const Source<kMultiTiled, RG>& src, const Seg& sg) {
    seq = src.table_row(p, sg.s);
    pos0 = src.pos0(p, sg.s);
    j = sg.j0;
    jend = sg.j0 + sg.n;
    len = sg.len;
  }
  struct Chunk {
    int j, nblk, ntok;
  };
  __device__ __forceinline__ Chunk next() {
    Chunk c;
    c.j = j;
    c.nblk = min(CB, jend - j);
    c.ntok = min(c.nblk * B, len - j * B);
    j += c.nblk;
    return c;
  }
};

template <bool kBf16, int G, int B>
__global__ void __launch_bounds__(kThreads, 1)
    pa_prefill_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap map_q,
                         const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
  constexpr int RG = kRows / G;  // positions per unit
  using Gm = Blk<B>;
  constexpr int CB = Gm::CB;
  const Source<kMultiTiled, RG> src;
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long cta = blockIdx.x;
  const int Hkv = p.num_kv_heads;

  // ---- set-up that reads no input
  if (tid == 0) {
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sm.kfull[i], 1);
      mbar_init(&sm.kempty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sm.vfull[i], 1);
      mbar_init(&sm.vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.qfull[i], 1);
      mbar_init(&sm.qempty[i], 1);
      mbar_init(&sm.mma_done[i], 1);
    }
    for (int i = 0; i < kOBufs; ++i) {
      mbar_init(&sm.unit_done[i], 1);
      mbar_init(&sm.o_free[i], 8);  // one arrival per softmax warp
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 8);
      mbar_init(&sm.pv_done[i], 1);
    }
    sm.abort = 0;
    sm.merge_ok = 0;
    sm.k_issued = sm.k_consumed = sm.v_issued = sm.v_consumed = sm.q_issued = sm.q_consumed = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
  }
  if (warp == kQKWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const volatile int* abort_flag = &sm.abort;

  // ---- inputs may come from the previous kernel in the stream
  grid_dependency_wait();
  grid_launch_dependents();
  zero_empty_units<kMultiTiled, RG, B>(p, src);
  WorkRange wr;
  Cursor cur;
  const bool has_work = decode_prologue<kThreads, B, CB>(p, sm.range, wr, cur, src);

  if (!has_work) {
    // nothing to stream
  } else if (warp == 0 || warp == kVWarp) {
    // ===================== producers ========================================
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    const bool is_k = warp == 0;
    // a sequence's K/V is reread by its other tiles: kept in L2 a while
    const uint64_t pol_kv = l2_policy_evict_last();
    const uint64_t pol_q = l2_policy_evict_first();
    bool ok = true;
    int ci = 0, qi = 0, k_issued = 0, v_issued = 0, q_issued = 0;
    if (p.test_flags & kFlagTestWithholdCopies) {
      if (lane == 0) {
        const uint64_t t0 = global_timer_ns();
        while (*abort_flag == 0 && global_timer_ns() - t0 < 4 * p.wait_limit_ns) {
        }
      }
      __syncwarp();
    } else {
      Seg sg;
      while (ok && next_seg<B, CB>(cur, sg, p, src)) {
        const int qs = qi & 1;
        if (is_k && lane == 0) {
          ok = mbar_wait_bounded(&sm.qempty[qs], ((qi >> 1) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
          if (ok) {
            // q rows: heads [h G, h G + G) of positions [z, z + RG), one box per head_dim half
            const int z = src.row_group0(p, sg.s);
            mbar_arrive_expect_tx(&sm.qfull[qs], kQBytes);
            tma_load_3d(sm.q[qs], &map_q, 0, sg.h * G, z, &sm.qfull[qs], pol_q);
            tma_load_3d(sm.q[qs] + kQHalf, &map_q, 64, sg.h * G, z, &sm.qfull[qs], pol_q);
            ++q_issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ++qi;
        Walk<RG, B> walk;
        walk.start(p, src, sg);
        const int32_t* trow = p.block_tables + static_cast<size_t>(walk.seq) * p.max_nb;
        // lane l < CB: entry of the chunk's block l, one chunk ahead
        typename Walk<RG, B>::Chunk cs = walk.next();
        int e_cur = lane < cs.nblk ? __ldg(trow + cs.j + lane) : 0;
        for (int c0 = 0; ok && c0 < sg.n; c0 += CB) {
          typename Walk<RG, B>::Chunk cn = cs;
          int e_next = 0;
          if (c0 + CB < sg.n) {
            cn = walk.next();
            e_next = lane < cn.nblk ? __ldg(trow + cn.j + lane) : 0;
          }
          int e = e_cur;
          if (lane < cs.nblk && (e < 0 || e >= p.num_blocks)) {
            record_status(p.status, PA_DEV_BAD_BLOCK_ID);
            e = 0;
          }
          const int ns = is_k ? kKStages : kVStages;
          const int st = ci % ns;
          uint64_t* empty = is_k ? &sm.kempty[st] : &sm.vempty[st];
          uint64_t* full = is_k ? &sm.kfull[st] : &sm.vfull[st];
          bool go = true;
          if (lane == 0) {
            go = mbar_wait_bounded(empty, ((ci / ns) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
            if (go) mbar_arrive_expect_tx(full, cs.nblk * Gm::kVBlockBytes);
          }
          ok = __shfl_sync(0xffffffffu, go, 0);
          if (!ok) break;
          if (lane < cs.nblk) {
            const int y = (e * Hkv + sg.h) * B;
            if (is_k && !Gm::kK3D) {
              uint8_t* base = sm.kbuf[st] + lane * Gm::kBlockBytes;
              tma_load_2d(base, &map_k, 0, y, full, pol_kv);
              tma_load_2d(base + kKHalf, &map_k, 64, y, full, pol_kv);
            } else {
              uint8_t* buf = is_k ? sm.kbuf[st] : sm.vbuf[st];
              tma_load_3d(buf + lane * Gm::kVBlockBytes, is_k ? &map_k : &map_v, 0, y, 0, full, pol_kv);
            }
          }
          __syncwarp();
          if (is_k) {
            ++k_issued;
          } else {
            ++v_issued;
          }
          ++ci;
          cs = cn;
          e_cur = e_next;
        }
      }
    }
    if (lane == 0) {
      if (is_k) {
        sm.k_issued = k_issued;
        sm.q_issued = q_issued;
      } else {
        sm.v_issued = v_issued;
      }
      if (!ok) {
        sm.abort = 1;
        record_status(p.status, PA_DEV_TIMEOUT);
      }
    }
  } else if (warp == kQKWarp) {
    // ===================== QK issuer =========================================
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    if (lane == 0) {
      constexpr uint32_t kIdescQK = make_idesc(kBf16, false, false, kChunk);  // q: K-major A, K: K-major B
      bool ok = true;
      int qk = 0, seg_i = 0;
      Seg sg;
      while (ok && next_seg<B, CB>(cur, sg, p, src)) {
        const int qs = seg_i & 1;
        ok = mbar_wait_bounded(&sm.qfull[qs], (seg_i >> 1) & 1, abort_flag, p.wait_limit_ns);
        const uint32_t q0 = smem_u32(sm.q[qs]);
        for (int c0 = 0; ok && c0 < sg.n; c0 += CB) {
          const int ks = qk % kKStages;
          const int sbuf = qk % kSBufs;
          ok = mbar_wait_bounded(&sm.kfull[ks], (qk / kKStages) & 1, abort_flag, p.wait_limit_ns) &&
               mbar_wait_bounded(&sm.pv_done[sbuf], ((qk / kSBufs) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k0 = smem_u32(sm.kbuf[ks]);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t a = sw128_desc(q0 + (k >> 2) * kQHalf + (k & 3) * 32, 16, 8 * kRowBytes);
            const uint64_t b = sw128_desc(k0 + (k >> 2) * Gm::kKHalfBytes + (k & 3) * 32, 16, Gm::kKGroupBytes);
            umma(tmem + kColS + sbuf * kChunk, a, b, kIdescQK, k > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full[sbuf]);
          umma_commit(&sm.kempty[ks]);
          ++qk;
        }
        if (!ok) break;
        umma_commit(&sm.qempty[qs]);  // q may be reloaded once the unit's last QK is done
        ++seg_i;
      }
      umma_commit(&sm.mma_done[0]);
      (void)mbar_wait_bounded(&sm.mma_done[0], 0, nullptr, p.wait_limit_ns);
      sm.k_consumed = qk;
      sm.q_consumed = seg_i;
      if (!ok) {
        sm.abort = 1;
        record_status(p.status, PA_DEV_TIMEOUT);
      }
    }
    __syncwarp();
  } else if (warp == kPVWarp) {
    // ===================== PV issuer =========================================
    // Per chunk, once its P is written (over its S, in TMEM) and its V has
    // landed: P head then P residual times V, for the 16-token steps that
    // hold valid tokens, into the unit's O buffer (unit i takes buffer
    // i % kOBufs, once the finish of the unit before has read it).  A comes
    // from TMEM: the 16 tokens of step k are 8 columns (two 16-bit values a
    // column) of the head's or the residual's 16 columns in the half of the
    // chunk's 128 columns that holds them.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    if (lane == 0) {
      constexpr uint32_t kIdescPV = make_idesc(kBf16, false, true, D);  // P: K-major A (TMEM), V: MN-major B
      bool ok = true;
      int pv = 0, seg_i = 0;
      Seg sg;
      while (ok && next_seg<B, CB>(cur, sg, p, src)) {
        Walk<RG, B> walk;
        walk.start(p, src, sg);
        const int ob = seg_i % kOBufs;
        ok = mbar_wait_bounded(&sm.o_free[ob], ((seg_i / kOBufs) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
        for (int c0 = 0; ok && c0 < sg.n; c0 += CB) {
          const int ntok = walk.next().ntok;
          const int vs = pv % kVStages;
          const int sbuf = pv % kSBufs;
          ok = mbar_wait_bounded(&sm.p_full[sbuf], (pv / kSBufs) & 1, abort_flag, p.wait_limit_ns) &&
               mbar_wait_bounded(&sm.vfull[vs], (pv / kVStages) & 1, abort_flag, p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v0 = smem_u32(sm.vbuf[vs]);
          const uint32_t pcol = tmem + kColS + sbuf * kChunk;
          const int nks = (ntok + 15) / 16;
          for (int k = 0; k < nks; ++k) {
            const uint64_t b = sw128_desc(v0 + Gm::v_offset(16 * k), Gm::kBlockBytes, Gm::kVGroupBytes);
            constexpr int kSteps = kHalfChunk / 16;  // 16-token steps in a warpgroup's half
            const uint32_t a_head = pcol + (k / kSteps) * kHalfChunk + (k % kSteps) * 8;
            umma_tmem_a(tmem + kColO + ob * D, a_head, b, kIdescPV, (c0 > 0 || k > 0) ? 1u : 0u);
            umma_tmem_a(tmem + kColO + ob * D, a_head + kHalfChunk / 2, b, kIdescPV, 1u);
          }
          umma_commit(&sm.pv_done[sbuf]);
          umma_commit(&sm.vempty[vs]);
          ++pv;
        }
        if (!ok) break;
        umma_commit(&sm.unit_done[ob]);
        ++seg_i;
      }
      umma_commit(&sm.mma_done[1]);
      (void)mbar_wait_bounded(&sm.mma_done[1], 0, nullptr, p.wait_limit_ns);
      sm.v_consumed = pv;
      if (!ok) {
        sm.abort = 1;
        record_status(p.status, PA_DEV_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    // ===================== softmax (warps 4..11) ============================
    // Thread r of warpgroup w owns row r: tokens [64 w, 64 w + 64) of each
    // chunk's S and P (P's head and residual in the same 64 columns),
    // head_dim [64 w, 64 w + 64) of O at the unit's finish.  A row's max over a
    // chunk is put together from its two halves through shared memory, so
    // both warpgroups take the same reference max; everything else about a
    // row is the thread's own.
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // this thread's query row (TMEM lane)
    const int wg = (warp - 4) / 4;
    const int col0 = wg * kHalfChunk;
    const int d0 = wg * (D / 2);
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const bool leader = warp == 4 && lane == 0;
    const int G_off = r % G;         // head within the kv head's group
    const int pos_off = r / G;       // position within the unit
    bool ok = true;
    int ci = 0, si = 0;
    float m_ref = kNoMax, l_sum = 0.f;  // the row's reference max; the sum over this warpgroup's tokens
    int32_t* arrival = nullptr;         // a published piece's arrival, counted a chunk later

    // chunk j's PV has completed (its S buffer's barrier; it cannot have
    // moved on, since chunk j + kSBufs's PV needs a P this thread has not
    // written)
    auto wait_pv = [&](int j) -> bool {
      const bool w = mbar_wait_bounded(&sm.pv_done[j % kSBufs], (j / kSBufs) & 1, abort_flag, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      return true;
    };
    // every PV of unit i (O buffer i % kOBufs) has completed
    auto wait_unit = [&](int i) -> bool {
      const bool w = mbar_wait_bounded(&sm.unit_done[i % kOBufs], (i / kOBufs) & 1, abort_flag, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      return true;
    };
    auto o_addr = [&](int ob, int c) -> uint32_t { return tmem + lane_base + kColO + ob * D + c; };

    // Online softmax of chunk ci of a unit whose rows start at position
    // pos0 of a sequence of len tokens; its PV goes to O buffer ob.
    auto softmax_chunk = [&](int ci, const typename Walk<RG, B>::Chunk& ch, int len, int pos0, bool first,
                             int ob) -> bool {
      const int sbuf = ci % kSBufs;
      const int sb = ci & 1;  // parity of the max exchange buffer
      const uint32_t s_addr = tmem + lane_base + kColS + sbuf * kChunk + col0;  // this half of the row
      const bool w = mbar_wait_bounded(&sm.s_full[sbuf], (ci / kSBufs) & 1, abort_flag, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      // tokens [0, nv) of this warpgroup's half of the chunk are visible to
      // this row: the sequence's tokens up to lim (causal), none past the
      // chunk's end
      const int lim = len - p.q_len + pos0 + pos_off;
      const int nv = max(0, min(min(ch.ntok, lim - ch.j * B + 1) - col0, kHalfChunk));
      // d = score - base, one FFMA a token, masked by selection (most chunks
      // are whole for every row: no per-token test there).  The base is the
      // reference max, or 0 on a unit's first chunk, so that the chunk's max
      // score mx + base never cancels against the no-max-yet sentinel.  S
      // comes in two loads of half the columns, the second in flight while
      // the first is scaled.
      const float m_base = first ? 0.f : m_ref;
      constexpr int kQ = kHalfChunk / 2;
      float s[kHalfChunk];
      uint32_t raw[kHalfChunk];
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nb2 = make_float2(-m_base, -m_base);
      float mxa = -INFINITY, mxb = -INFINITY;  // two partial maxima: two dependency chains
      // whether any row of the warp has masked tokens here (the chunks on a
      // unit's causal diagonal or at its sequence's end): the masking is
      // then taken by the whole warp, and skipped by it otherwise
      const bool masked = __any_sync(0xffffffffu, nv != kHalfChunk);
      tmem_ld_nowait<kQ>(s_addr, raw);
      tmem_wait_ld();
      tmem_ld_nowait<kQ>(s_addr + kQ, raw + kQ);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        if (part == 1) tmem_wait_ld();
        if (masked) {
#pragma unroll
          for (int c = part * kQ; c < (part + 1) * kQ; c += 2) {
            float2 d = fma2(make_float2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), sc2, nb2);
            d.x = c < nv ? d.x : -INFINITY;
            d.y = c + 1 < nv ? d.y : -INFINITY;
            s[c] = d.x;
            s[c + 1] = d.y;
            if ((c >> 1) & 1) {
              mxb = max3(mxb, d.x, d.y);
            } else {
              mxa = max3(mxa, d.x, d.y);
            }
          }
        } else {
#pragma unroll
          for (int c = part * kQ; c < (part + 1) * kQ; c += 2) {
            const float2 d = fma2(make_float2(__uint_as_float(raw[c]), __uint_as_float(raw[c + 1])), sc2, nb2);
            s[c] = d.x;
            s[c + 1] = d.y;
            if ((c >> 1) & 1) {
              mxb = max3(mxb, d.x, d.y);
            } else {
              mxa = max3(mxa, d.x, d.y);
            }
          }
        }
      }
      float mx = fmaxf(mxa, mxb);
      // the row's max over the whole chunk: this half's and the other's
      sm.red[sb][wg][r] = mx;
      named_barrier_sync(kPairBarrier, 256);
      mx = fmaxf(mx, sm.red[sb][wg ^ 1][r]);
      // the reference max moves only when a score passes it by more than
      // kRescaleGap (always on a unit's first chunk); then d is shifted to
      // the new one and O's row is scaled by alpha.  Both warpgroups decide
      // alike for a row.  The step is taken by the warp as a whole: a row
      // that keeps its reference gets a shift of 0 and alpha = 1.
      const bool moves = first || mx > kRescaleGap;
      const bool any_moves = __any_sync(0xffffffffu, moves);
      float alpha = 1.f;
      if (any_moves) {
        const float m_old = first ? -INFINITY : m_ref;
        const float m_new = moves ? fmaxf(fmaxf(m_old, mx + m_base), kNoMax) : m_ref;  // mx + m_base: the chunk's max
        alpha = moves ? fast_exp2(m_old - m_new) : 1.f;
        l_sum = first ? 0.f : l_sum * alpha;
        const float2 shift = make_float2(m_base - m_new, m_base - m_new);
#pragma unroll
        for (int c = 0; c < kHalfChunk; c += 2) {
          const float2 d = add2(make_float2(s[c], s[c + 1]), shift);
          s[c] = d.x;
          s[c + 1] = d.y;
        }
        m_ref = m_new;
      }
      // this warpgroup's half of O's rows, once the previous PV is done, by
      // the warp as a whole (TMEM loads and stores are warp-wide): a row
      // whose reference stayed takes alpha = 1
      if (!first && any_moves) {
        if (!wait_pv(ci - 1)) return false;
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < D / 2; c += 32) {
          uint32_t o[32];
          tmem_ld_nowait<32>(o_addr(ob, d0 + c), o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 d = mul2(make_float2(__uint_as_float(o[k]), __uint_as_float(o[k + 1])), a2);
            o[k] = __float_as_uint(d.x);
            o[k + 1] = __float_as_uint(d.y);
          }
          tmem_st<32>(o_addr(ob, d0 + c), o);
        }
        tmem_wait_st();
      }
      // probabilities, and P over this half's S columns (read above): the
      // head in the first half of them, the residual in the second; the
      // first 32 tokens' columns go out while the rest are computed
      uint32_t hw[kHalfChunk / 2], lw[kHalfChunk / 2];
      float2 la = make_float2(0.f, 0.f), lb = la;  // partial row sums, two chains
#pragma unroll
      for (int part = 0; part < 2; ++part) {
#pragma unroll
        for (int k = part * kQ / 2; k < (part + 1) * kQ / 2; ++k) {
          const float a0 = fast_exp2(s[2 * k]), a1 = fast_exp2(s[2 * k + 1]);  // 0 when masked
          if (k & 1) {
            lb = add2(lb, make_float2(a0, a1));
          } else {
            la = add2(la, make_float2(a0, a1));
          }
          split_pair<kBf16>(a0, a1, hw[k], lw[k]);
        }
        tmem_st<kQ / 2>(s_addr + part * kQ / 2, hw + part * kQ / 2);
        tmem_st<kQ / 2>(s_addr + kHalfChunk / 2 + part * kQ / 2, lw + part * kQ / 2);
      }
      la = add2(la, lb);
      l_sum += la.x + la.y;
      // V rows past the sequence end inside the last 16-token step are
      // zeroed so that 0 * (whatever they hold) cannot reach the output
      // (thread r of the first warpgroup takes token row r)
      if (wg == 0 && r >= ch.ntok && r < ((ch.ntok + 15) & ~15)) {
        const int vs = ci % kVStages;
        (void)mbar_wait_bounded(&sm.vfull[vs], (ci / kVStages) & 1, abort_flag, p.wait_limit_ns);
        uint4* v0 = reinterpret_cast<uint4*>(sm.vbuf[vs] + Gm::v_offset(r));
        uint4* v1 = reinterpret_cast<uint4*>(sm.vbuf[vs] + Gm::v_offset(r) + Gm::kBlockBytes);
#pragma unroll
        for (int i = 0; i < kRowBytes / 16; ++i) {
          v0[i] = make_uint4(0, 0, 0, 0);
          v1[i] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[sbuf]);
      return true;
    };

    // The finish of a unit whose PVs have all completed: its rows' outputs,
    // its published partial state, or (its first piece) the merge of every
    // piece.  m is the row's reference max, l this warpgroup's part of its
    // sum; s_seq, pos0 the unit's sequence and first position; ob its O
    // buffer, handed back after.  Each warpgroup takes its 64 head_dim
    // columns.
    auto finish_unit = [&](const Seg& fs, float m, float l, int s_seq, int pos0, int ob) {
      const int pos = pos0 + pos_off;
      const bool real = pos < p.q_len;
      uint16_t* out_row =
          p.out + ((static_cast<size_t>(s_seq) * p.q_len + pos) * p.num_q_heads + fs.h * G + G_off) * D + d0;
      // this warpgroup's half of O's row, loaded at once (in flight while
      // the row sums are exchanged); the O buffer is handed back as soon as
      // it has been read
      float a[D / 2];
      {
        uint32_t o[D / 2];
        tmem_ld_nowait<32>(o_addr(ob, d0), o);
        tmem_ld_nowait<32>(o_addr(ob, d0 + 32), o + 32);
        sm.lsum[wg][r] = l;
        named_barrier_sync(kPairBarrier, 256);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < D / 2; ++k) a[k] = __uint_as_float(o[k]);
      }
      const float L = sm.lsum[0][r] + sm.lsum[1][r];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free[ob]);
      // the row's outputs: 64 columns, 16-bit, rounded to nearest even
      auto store_row = [&]() {
        if (!real) return;
        uint32_t w[D / 4];
#pragma unroll
        for (int k = 0; k < D / 4; ++k) w[k] = pack2<kBf16>(a[2 * k], a[2 * k + 1]);
        uint4* o = reinterpret_cast<uint4*>(out_row);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) o[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
      };
      auto scale_row = [&](float f) {
        const float2 f2 = make_float2(f, f);
#pragma unroll
        for (int k = 0; k < D / 2; k += 2) {
          const float2 v = mul2(make_float2(a[k], a[k + 1]), f2);
          a[k] = v.x;
          a[k + 1] = v.y;
        }
      };
      const bool opens = fs.j0 == fs.first, closes = fs.j0 + fs.n == fs.nb;
      if (opens && closes) {
        scale_row(L > 0.f ? __fdividef(1.f, L) : 0.f);  // L >= 1 for a row that saw a token
        store_row();
      } else if (!opens) {
        // publish m, l and the row of O; the arrival is counted after the
        // next chunk, once these stores have drained
        float* pp = p.partials + partial_slot(cta, fs.unit_first, wr) * kPartStride;
        if (wg == 0) {
          pp[r] = m;
          pp[kRows + r] = L;
        }
        float4* pa = reinterpret_cast<float4*>(pp + 2 * kRows + r * D + d0);
#pragma unroll
        for (int k = 0; k < D / 8; ++k) pa[k] = make_float4(a[4 * k], a[4 * k + 1], a[4 * k + 2], a[4 * k + 3]);
        named_barrier_sync(kPairBarrier, 256);
        if (leader) arrival = unit_counter(p, fs);
      } else {
        // merge: pieces first + 1 .. last were published by the CTAs after this one
        const long long last = cta_of(fs.unit_last, wr.total, wr.nparts);
        const uint32_t need = static_cast<uint32_t>(last - cta);
        int32_t* counter = unit_counter(p, fs);
        if (leader) {
          const bool got = wait_arrivals(counter, 0, need, p.wait_limit_ns);
          if (got) {
            atomicSub(reinterpret_cast<unsigned int*>(counter), need);  // back to zero for the next launch
          } else {
            record_status(p.status, PA_DEV_TIMEOUT);
          }
          sm.merge_ok = got;
        }
        named_barrier_sync(kPairBarrier, 256);
        if (sm.merge_ok) {
          float M = m;
          for (long long cc = cta + 1; cc <= last; ++cc) {
            M = fmaxf(M, __ldcg(p.partials + partial_slot(cc, fs.unit_first, wr) * kPartStride + r));
          }
          float Lt = L * fast_exp2(m - M);
          for (long long cc = cta + 1; cc <= last; ++cc) {
            const float* pp = p.partials + partial_slot(cc, fs.unit_first, wr) * kPartStride;
            Lt = fmaf(__ldcg(pp + kRows + r), fast_exp2(__ldcg(pp + r) - M), Lt);
          }
          const float inv = Lt > 0.f ? __fdividef(1.f, Lt) : 0.f;
          scale_row(fast_exp2(m - M) * inv);
          for (long long cc = cta + 1; cc <= last; ++cc) {
            const float* pp = p.partials + partial_slot(cc, fs.unit_first, wr) * kPartStride;
            const float wb = fast_exp2(__ldcg(pp + r) - M) * inv;
            const float4* pa = reinterpret_cast<const float4*>(pp + 2 * kRows + r * D + d0);
#pragma unroll
            for (int k = 0; k < D / 8; ++k) {
              const float4 v = __ldcg(pa + k);
              a[4 * k] = fmaf(v.x, wb, a[4 * k]);
              a[4 * k + 1] = fmaf(v.y, wb, a[4 * k + 1]);
              a[4 * k + 2] = fmaf(v.z, wb, a[4 * k + 2]);
              a[4 * k + 3] = fmaf(v.w, wb, a[4 * k + 3]);
            }
          }
          store_row();
        }
      }
    };
    auto count_arrival = [&]() {
      if (arrival != nullptr) {
        __threadfence();
        atomicAdd(reinterpret_cast<unsigned int*>(arrival), 1u);
        arrival = nullptr;
      }
    };

    Seg sg, prev;
    float prev_m = 0.f, prev_l = 0.f;
    int prev_seq = 0, prev_pos0 = 0;
    bool have_prev = false;
    while (ok && next_seg<B, CB>(cur, sg, p, src)) {
      Walk<RG, B> walk;
      walk.start(p, src, sg);
      const int ob = si % kOBufs;
      for (int c0 = 0; c0 < sg.n; c0 += CB) {
        if (c0 == 0 && have_prev) {  // the previous unit's state, before this one resets it
          prev_m = m_ref;
          prev_l = l_sum;
        }
        ok = softmax_chunk(ci, walk.next(), walk.len, walk.pos0, c0 == 0, ob);
        if (!ok) break;
        ++ci;
        if (leader) count_arrival();
        if (c0 == 0 && have_prev) {
          ok = wait_unit(si - 1);  // every PV of the previous unit
          if (!ok) break;
          finish_unit(prev, prev_m, prev_l, prev_seq, prev_pos0, (si - 1) % kOBufs);
          have_prev = false;
        }
      }
      if (!ok) break;
      prev = sg;
      prev_seq = walk.seq;
      prev_pos0 = walk.pos0;
      have_prev = true;
      ++si;
    }
    if (ok && have_prev) {
      ok = wait_unit(si - 1);
      if (ok) finish_unit(prev, m_ref, l_sum, prev_seq, prev_pos0, (si - 1) % kOBufs);
    }
    if (leader) count_arrival();
    if (!ok && lane == 0) {
      sm.abort = 1;
      record_status(p.status, PA_DEV_TIMEOUT);
    }
  }

  // ---- teardown: drain copies after an abort, release TMEM
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0 && sm.abort) {
    for (int k = sm.k_consumed; k < sm.k_issued; ++k) {
      (void)mbar_wait_bounded(&sm.kfull[k % kKStages], (k / kKStages) & 1, nullptr, p.wait_limit_ns);
    }
    for (int k = sm.v_consumed; k < sm.v_issued; ++k) {
      (void)mbar_wait_bounded(&sm.vfull[k % kVStages], (k / kVStages) & 1, nullptr, p.wait_limit_ns);
    }
    for (int k = sm.q_consumed; k < sm.q_issued; ++k) {
      (void)mbar_wait_bounded(&sm.qfull[k & 1], (k >> 1) & 1, nullptr, p.wait_limit_ns);
    }
  }
  if (warp == kQKWarp) tmem_dealloc(tmem, kTmemCols);
}

// ---- host side -----------------------------------------------------------------

template <bool kBf16, int G, int B>
cudaError_t launch_prefill(const Variant& v, const DecodeParams& prm, int ctas, cudaStream_t stream) {
  constexpr int RG = kRows / G;
  CUtensorMap mq, mk, mv;
  const unsigned long long q_rows = static_cast<unsigned long long>(prm.num_seqs) * prm.q_len;
  const unsigned long long kv_rows = static_cast<unsigned long long>(prm.num_blocks) * prm.num_kv_heads * B;
  if (kv_rows >= (1ull << 31) || q_rows >= (1ull << 31)) return cudaErrorInvalidValue;
  LaunchMaps want{};
  want.kernel = reinterpret_cast<const void*>(&pa_prefill_tc_kernel<kBf16, G, B>);
  want.q = prm.q;
  want.k = prm.k_pool;
  want.v = prm.v_pool;
  want.q_rows = q_rows;
  want.kv_rows = kv_rows;
  want.num_q_heads = prm.num_q_heads;
  if (!cached_maps(want, mq, mk, mv, &encode_launch_maps<kBf16, G, RG, B>)) return cudaErrorInvalidValue;
  // setmaxnreg only moves registers inside the launch's allocation; should a
  // build give the kernel fewer than the split needs, the softmax warps'
  // increase would wait forever, so such a kernel is not launched
  static const bool regs_fit = [] {
    cudaFuncAttributes a{};
    return cudaFuncGetAttributes(&a, pa_prefill_tc_kernel<kBf16, G, B>) == cudaSuccess &&
           a.numRegs * kThreads >= 128 * kCtrlRegs + 256 * kSoftmaxRegs;
  }();
  if (!regs_fit) return cudaErrorInvalidConfiguration;
  return launch_overlapped(pa_prefill_tc_kernel<kBf16, G, B>, dim3(ctas), dim3(kThreads),
                           static_cast<size_t>(v.smem_bytes), stream, prm, mq, mk, mv);
}

// Partition cost of finishing a 128-row unit, in 1/8 of a 128-token chunk.
constexpr int kUnitCost = 8;

template <bool kBf16, int G, int B>
Variant prefill_variant() {
  return Variant{reinterpret_cast<const void*>(&pa_prefill_tc_kernel<kBf16, G, B>), kThreads, smem_bytes(),
                 kPartStride, &launch_prefill<kBf16, G, B>, kUnitCost};
}

template <bool kBf16, int B>
bool pick(int G, Variant& v) {
  switch (G) {
    case 1: v = prefill_variant<kBf16, 1, B>(); return true;
    case 2: v = prefill_variant<kBf16, 2, B>(); return true;
    case 4: v = prefill_variant<kBf16, 4, B>(); return true;
    case 8: v = prefill_variant<kBf16, 8, B>(); return true;
    default: return false;
  }
}

}  // namespace pf
}  // namespace tc
}  // namespace pa
