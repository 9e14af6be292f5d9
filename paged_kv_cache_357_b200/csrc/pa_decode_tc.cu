// pa_decode tensor-core kernel (tcgen05 + TMEM + TMA), sm_100a.
//
// Same computation as the CUDA-core kernel (vLLM blog §"关键细节" 2): out =
// softmax(scale * q K^T) V over each sequence's paged tokens, merged across
// blocks with a running max and sum (PagedAttention study notes ch.05 §4).
// Used where a GQA group of G = 4 or 8 query heads shares each kv head, which
// makes both products real (if thin) matrix products:
//
//   S^T[token, head] = K_chunk[token, :] . Q^T[:, head]      (M=128, N=16, K=128)
//   O^T[d, head]     = V_chunk^T[d, token] . P^T[token, head] (M=128, N=16, K=16 per step)
//
// N = 16 covers the G heads of the group (the other columns are computed and
// ignored).  A chunk is up to 8 blocks (128 tokens) of one (sequence, kv head)
// unit; the work partition over CTAs is the one in pa_decode_common.cuh.
//
// Roles (192 threads, one CTA per SM):
//   warp 0      producer: resolves block ids, issues 2-D TMA loads of the K and
//               V tiles (64-column boxes, 128-byte swizzle) into separate rings
//               of 32 KB chunk stages — 2 for K, released when its QK is done,
//               4 for V, released when its PV is done — and of the q rows.
//   warp 1      allocates 64 TMEM columns; lane 0 issues every tcgen05.mma and
//               tcgen05.commit, polling which of QK(next) and PV(oldest
//               pending) is ready and issuing it.
//   warps 2-5   softmax + epilogue, one TMEM lane (token row, then head_dim
//               index) per thread: read S^T from TMEM, online softmax with a
//               cross-warp max per chunk, write P^T (bf16/fp16) into a swizzled
//               shared buffer, zero V rows past the sequence end inside the
//               last 16-token step, then read O^T and rescale-accumulate.
//               The epilogue of chunk i runs after the softmax of chunk i+1.
// The swizzled layouts written by TMA serve both products directly: the K
// tile is a K-major A operand for QK, the V tile an MN-major A operand for PV.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "pa_decode_host.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace tc {

constexpr int D = 128;
constexpr int B = 16;
constexpr int kChunkTok = 128;             // tokens per chunk = MMA M of QK
constexpr int CB = kChunkTok / B;          // blocks per chunk
constexpr int N = 16;                      // MMA N (query heads, padded)
constexpr int kKStages = 2;  // K is released as soon as its QK completes
constexpr int kVStages = 4;  // V is held until its PV completes
constexpr int kRowBytes = 128;             // one swizzle row: 64 elements
constexpr int kHalfBytes = kChunkTok * kRowBytes;  // 64 head_dim columns x 128 tokens
constexpr int kOperandBytes = 2 * kHalfBytes;      // head_dim [0:64) then [64:128)
constexpr int kBlockBytes = B * kRowBytes;         // one block's rows in one half
constexpr int kQSlotBytes = 2 * N * kRowBytes;     // two halves of 16 rows
constexpr int kPSlotBytes = 2 * N * kRowBytes;     // tokens [0,64) and [64,128), 16 rows each
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kSoftmaxBarrier = 1;
constexpr uint32_t kTmemCols = 64;  // S[0], S[1], O[0], O[1]: 16 fp32 columns each

struct TcSmem {
  uint8_t kbuf[kKStages][kOperandBytes];  // 1024-aligned regions
  uint8_t vbuf[kVStages][kOperandBytes];
  uint8_t q[2][kQSlotBytes];
  uint8_t p[2][kPSlotBytes];
  float red[2][4][8];
  float lred[4][8];
  uint64_t kfull[kKStages];
  uint64_t kempty[kKStages];
  uint64_t vfull[kVStages];
  uint64_t vempty[kVStages];
  uint64_t qfull[2];
  uint64_t qempty[2];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t o_free[2];
  uint64_t mma_done;
  RangeSmem range;
  uint32_t tmem_base;
  int abort;
  int is_last;
  int k_issued;
  int k_consumed;
  int v_issued;
  int v_consumed;
  int q_issued;
  int q_consumed;
};
constexpr int kSmemBytes = static_cast<int>(sizeof(TcSmem)) + 1024;  // + alignment slack

// ---- tcgen05 / TMA primitives ------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] . B[smem desc], kind::f16, fp32 accumulate.
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  setp.ne.b32 p, %4, 0;\n"
      "  tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version 1.
// lbo/sbo in bytes: lbo = distance between 64-element column groups of an
// MN-major operand (unused for K-major), sbo = distance between 8-row groups.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulate, A/B both bf16 or both
// fp16, B K-major, A K-major (QK) or MN-major (PV), M = 128, N = 16.
__host__ __device__ constexpr uint32_t make_idesc(bool bf16, bool a_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

struct ChunkInfo {
  int j;     // first logical block of the chunk in its unit
  int nblk;  // blocks in the chunk
  int ntok;  // valid tokens in the chunk
};

__device__ __forceinline__ ChunkInfo chunk_at(const Seg& sg, int c0) {
  ChunkInfo c;
  c.j = sg.j0 + c0;
  c.nblk = min(CB, sg.n - c0);
  c.ntok = min(c.nblk * B, sg.len - c.j * B);
  return c;
}

template <bool kBf16, int G>
__global__ void __launch_bounds__(kThreads, 1)
    pa_decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap map_q,
                        const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
  static_assert(G == 4 || G == 8, "tensor-core decode covers groups of 4 and 8");
  extern __shared__ unsigned char smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long cta = blockIdx.x;
  const int Hq = p.num_q_heads, Hkv = p.num_kv_heads;

  // ---- set-up that reads no input (barriers, TMEM, tensor-map prefetch);
  // with programmatic dependent launch it overlaps the previous kernel
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
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 4);
      mbar_init(&sm.p_full[i], 4);
      mbar_init(&sm.o_full[i], 1);
      mbar_init(&sm.o_free[i], 4);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    sm.k_issued = 0;
    sm.k_consumed = 0;
    sm.v_issued = 0;
    sm.v_consumed = 0;
    sm.q_issued = 0;
    sm.q_consumed = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const volatile int* abort_flag = &sm.abort;
  constexpr uint32_t kColS = 0, kColO = 32;

  // ---- inputs may come from the previous kernel in the stream
  grid_dependency_wait();
  grid_launch_dependents();
  zero_empty_outputs<kThreads, B>(p, D);
  WorkRange wr;
  Cursor cur;
  const bool has_work = decode_prologue<kThreads, B, CB>(p, sm.range, wr, cur);  // uniform across the CTA

  if (!has_work) {
    // nothing to stream: straight to teardown
  } else if (warp == 0) {
    // ===================== producer =========================================
    const uint64_t pol_stream = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();
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
      while (ok && next_seg<B, CB>(cur, sg, p)) {
        const int qs = qi & 1;
        if (lane == 0) {
          ok = mbar_wait_bounded(&sm.qempty[qs], ((qi >> 1) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
          if (ok) {
            const int y = sg.s * Hq + sg.h * G;
            mbar_arrive_expect_tx(&sm.qfull[qs], kQSlotBytes);
            tma_load_2d(sm.q[qs], &map_q, 0, y, &sm.qfull[qs], pol_keep);
            tma_load_2d(sm.q[qs] + N * kRowBytes, &map_q, 64, y, &sm.qfull[qs], pol_keep);
            ++q_issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ++qi;
        // Block-table entries 32 at a time (lane l holds entry b0 + l); the
        // next batch is in flight while the current one is issued.
        const int32_t* trow = p.block_tables + static_cast<size_t>(sg.s) * p.max_nb + sg.j0;
        int e_cur = (lane < sg.n) ? __ldg(trow + lane) : 0;
        for (int b0 = 0; ok && b0 < sg.n; b0 += 32) {
          const int e_next = (b0 + 32 + lane < sg.n) ? __ldg(trow + b0 + 32 + lane) : 0;
          if (b0 + lane < sg.n && (e_cur < 0 || e_cur >= p.num_blocks)) {
            record_status(p.status, PA_DEV_BAD_BLOCK_ID);
            e_cur = 0;
          }
          const int b_end = min(b0 + 32, sg.n);
          for (int c0 = b0; c0 < b_end; c0 += CB) {
            const ChunkInfo ch = chunk_at(sg, c0);
            const int e = __shfl_sync(0xffffffffu, e_cur, (c0 - b0) + (lane & (CB - 1)));
            const int ks = ci % kKStages, vs = ci % kVStages;
            const int y = (e * Hkv + sg.h) * B;
            if (lane == 0) {
              ok = mbar_wait_bounded(&sm.kempty[ks], ((ci / kKStages) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
              if (ok) mbar_arrive_expect_tx(&sm.kfull[ks], ch.nblk * 2 * kBlockBytes);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane < ch.nblk) {
              uint8_t* base = sm.kbuf[ks] + lane * kBlockBytes;
              tma_load_2d(base, &map_k, 0, y, &sm.kfull[ks], pol_stream);
              tma_load_2d(base + kHalfBytes, &map_k, 64, y, &sm.kfull[ks], pol_stream);
            }
            __syncwarp();
            ++k_issued;
            if (lane == 0) {
              ok = mbar_wait_bounded(&sm.vempty[vs], ((ci / kVStages) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
              if (ok) mbar_arrive_expect_tx(&sm.vfull[vs], ch.nblk * 2 * kBlockBytes);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane < ch.nblk) {
              uint8_t* base = sm.vbuf[vs] + lane * kBlockBytes;
              tma_load_2d(base, &map_v, 0, y, &sm.vfull[vs], pol_stream);
              tma_load_2d(base + kHalfBytes, &map_v, 64, y, &sm.vfull[vs], pol_stream);
            }
            __syncwarp();
            ++v_issued;
            ++ci;
          }
          e_cur = e_next;
        }
      }
    }
    if (lane == 0) {
      sm.k_issued = k_issued;
      sm.v_issued = v_issued;
      sm.q_issued = q_issued;
      if (!ok) {
        sm.abort = 1;
        record_status(p.status, PA_DEV_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer ========================================
    // A non-blocking scheduler: each pass tests whether QK of the next chunk
    // (its K/V landed, its S buffer free, its q ready) or PV of the oldest
    // chunk still waiting (its P written, its O buffer free) can go, and
    // issues whichever can, so PV of chunk i never waits for chunk i+1's data.
    if (lane == 0) {
      constexpr uint32_t kIdescQK = make_idesc(kBf16, false);
      constexpr uint32_t kIdescPV = make_idesc(kBf16, true);
      bool ok = true;
      int qk = 0, pv = 0, seg_i = 0, q_consumed = 0;
      uint32_t ring = 0;  // valid tokens of each pending chunk (index & 3), 8 bits each
      bool have_seg = false, q_ready = false, walk_done = false;
      int c0 = 0;
      Seg sg;
      uint64_t t_idle = 0;
      uint32_t idle = 0;
      while (ok) {
        bool progress = false;
        if (!walk_done && !have_seg) {
          if (next_seg<B, CB>(cur, sg, p)) {
            have_seg = true;
            c0 = 0;
          } else {
            walk_done = true;
          }
        }
        if (have_seg) {
          const int qs = seg_i & 1;
          if (!q_ready && mbar_test_wait(&sm.qfull[qs], (seg_i >> 1) & 1)) {
            q_ready = true;
            ++q_consumed;
          }
          const int ks = qk % kKStages;
          if (q_ready && qk - pv < 4 && mbar_test_wait(&sm.kfull[ks], (qk / kKStages) & 1) &&
              mbar_test_wait(&sm.s_free[qk & 1], ((qk >> 1) & 1) ^ 1u)) {
            tc_fence_after();
            const uint32_t k0 = smem_u32(sm.kbuf[ks]);
            const uint32_t q0 = smem_u32(sm.q[qs]);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint64_t a = sw128_desc(k0 + (k >> 2) * kHalfBytes + (k & 3) * 32, 16, 8 * kRowBytes);
              const uint64_t b = sw128_desc(q0 + (k >> 2) * N * kRowBytes + (k & 3) * 32, 16, 8 * kRowBytes);
              umma(tmem + kColS + (qk & 1) * N, a, b, kIdescQK, k > 0 ? 1u : 0u);
            }
            umma_commit(&sm.s_full[qk & 1]);
            umma_commit(&sm.kempty[ks]);
            const int slot_shift = (qk & 3) * 8;
            ring = (ring & ~(0xFFu << slot_shift)) | (static_cast<uint32_t>(chunk_at(sg, c0).ntok) << slot_shift);
            c0 += CB;
            if (c0 >= sg.n) {  // last chunk of the segment: q may be reloaded after this QK
              umma_commit(&sm.qempty[qs]);
              have_seg = false;
              q_ready = false;
              ++seg_i;
            }
            ++qk;
            progress = true;
          }
        }
        if (pv < qk) {
          const int pb = pv & 1;
          const uint32_t par = (pv >> 1) & 1;
          const int vs = pv % kVStages;
          if (mbar_test_wait(&sm.p_full[pb], par) && mbar_test_wait(&sm.o_free[pb], par ^ 1u) &&
              mbar_test_wait(&sm.vfull[vs], (pv / kVStages) & 1)) {
            tc_fence_after();
            const int ntok = static_cast<int>((ring >> ((pv & 3) * 8)) & 0xFFu);
            const uint32_t v0 = smem_u32(sm.vbuf[vs]);
            const uint32_t p0 = smem_u32(sm.p[pb]);
            const int nks = (ntok + 15) / 16;
            for (int k = 0; k < nks; ++k) {
              const uint64_t a = sw128_desc(v0 + k * 16 * kRowBytes, kHalfBytes, 8 * kRowBytes);
              const uint64_t b = sw128_desc(p0 + (k >> 2) * N * kRowBytes + (k & 3) * 32, 16, 8 * kRowBytes);
              umma(tmem + kColO + pb * N, a, b, kIdescPV, k > 0 ? 1u : 0u);
            }
            umma_commit(&sm.o_full[pb]);
            umma_commit(&sm.vempty[vs]);
            ++pv;
            progress = true;
          }
        } else if (walk_done) {
          break;  // every chunk has had its QK and its PV
        }
        if (progress) {
          idle = 0;
        } else if ((++idle & 63u) == 0) {
          const uint64_t now = global_timer_ns();
          if (idle == 64) t_idle = now;
          if (*abort_flag != 0 || now - t_idle > p.wait_limit_ns) ok = false;
        }
      }
      // every MMA issued above completes before TMEM is released
      umma_commit(&sm.mma_done);
      (void)mbar_wait_bounded(&sm.mma_done, 0, nullptr, p.wait_limit_ns);
      sm.k_consumed = qk;
      sm.v_consumed = pv;
      sm.q_consumed = q_consumed;
      if (!ok) {
        sm.abort = 1;
        record_status(p.status, PA_DEV_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    // ===================== softmax + epilogue (warps 2-5) ====================
    // Per chunk i: softmax(i) then the epilogue of chunk i-1, so the PV of
    // chunk i-1 runs on the tensor core while the softmax of chunk i runs here.
    const int quad = warp & 3;           // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;      // token row of the chunk; head_dim index in the epilogue
    const int ctid = tid - 64;           // 0..127
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    int ci = 0;
    Seg sg;
    float m[G], lthr[G], acc[G], a_pend[G];

    // Online softmax of chunk ci; writes its P^T and returns the rescale
    // factor of the running output in alpha.
    auto softmax_chunk = [&](int ci, const ChunkInfo& ch, float* alpha) -> bool {
      const int vs = ci % kVStages;
      const int sb = ci & 1;
      const uint32_t par = (ci >> 1) & 1;
      bool w = mbar_wait_bounded(&sm.s_full[sb], par, abort_flag, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      float s16[16];
      tmem_ld16(tmem + lane_base + kColS + sb * N, s16);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free[sb]);

      const bool valid = r < ch.ntok;
      float sc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        sc[g] = valid ? s16[g] * p.scale_log2 : -INFINITY;
        float wm = sc[g];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) wm = fmaxf(wm, __shfl_xor_sync(0xffffffffu, wm, o));
        if (lane == 0) sm.red[sb][quad][g] = wm;
      }
      named_barrier_sync(kSoftmaxBarrier, kSoftmaxThreads);
      float pr[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float cm = fmaxf(fmaxf(sm.red[sb][0][g], sm.red[sb][1][g]), fmaxf(sm.red[sb][2][g], sm.red[sb][3][g]));
        const float m_new = fmaxf(m[g], cm);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[g] = fast_exp2(m[g] - m_use);
        m[g] = m_new;
        pr[g] = fast_exp2(sc[g] - m_use);
        lthr[g] = fmaf(lthr[g], alpha[g], pr[g]);
      }
      // P^T into the swizzled B operand: row = head, column = token
      const int pb = ci & 1;
      {
        uint8_t* pbase = sm.p[pb] + (r >> 6) * (N * kRowBytes);
        const int c = r & 63;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const int off = (g >> 3) * (8 * kRowBytes) + (g & 7) * kRowBytes + ((((c >> 3) ^ (g & 7)) & 7) << 4) +
                          (c & 7) * 2;
          const uint32_t two = pack2<kBf16>(pr[g], 0.f);
          *reinterpret_cast<uint16_t*>(pbase + off) = static_cast<uint16_t>(two & 0xffffu);
        }
      }
      // V rows past the sequence end inside the last 16-token step are zeroed
      // so that 0 * (whatever they hold) cannot reach the output
      if ((ch.ntok & 15) != 0 && r >= ch.ntok && r < ((ch.ntok + 15) & ~15)) {
        (void)mbar_wait_bounded(&sm.vfull[vs], (ci / kVStages) & 1, abort_flag, p.wait_limit_ns);
        uint4* v0 = reinterpret_cast<uint4*>(sm.vbuf[vs] + r * kRowBytes);
        uint4* v1 = reinterpret_cast<uint4*>(sm.vbuf[vs] + kHalfBytes + r * kRowBytes);
#pragma unroll
        for (int i = 0; i < kRowBytes / 16; ++i) {
          v0[i] = make_uint4(0, 0, 0, 0);
          v1[i] = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[pb]);
      return true;
    };

    // acc = acc * alpha + O^T row r of chunk ci.
    auto epilogue_chunk = [&](int ci, const float* alpha) -> bool {
      const int pb = ci & 1;
      bool w = mbar_wait_bounded(&sm.o_full[pb], (ci >> 1) & 1, abort_flag, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      float o16[16];
      tmem_ld16(tmem + lane_base + kColO + pb * N, o16);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free[pb]);
#pragma unroll
      for (int g = 0; g < G; ++g) acc[g] = fmaf(acc[g], alpha[g], o16[g]);
      return true;
    };

    while (ok && next_seg<B, CB>(cur, sg, p)) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        lthr[g] = 0.f;
        acc[g] = 0.f;
      }
      bool pending = false;
      for (int c0 = 0; c0 < sg.n; c0 += CB) {
        float alpha[G];
        ok = softmax_chunk(ci, chunk_at(sg, c0), alpha);
        if (!ok) break;
        if (pending) {
          ok = epilogue_chunk(ci - 1, a_pend);
          if (!ok) break;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) a_pend[g] = alpha[g];
        pending = true;
        ++ci;
      }
      if (ok && pending) ok = epilogue_chunk(ci - 1, a_pend);
      if (!ok) break;

      // ---- end of the segment: total sums, then output or partial state
      float L[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = lthr[g];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) sm.lred[quad][g] = v;
      }
      named_barrier_sync(kSoftmaxBarrier, kSoftmaxThreads);
#pragma unroll
      for (int g = 0; g < G; ++g) L[g] = (sm.lred[0][g] + sm.lred[1][g]) + (sm.lred[2][g] + sm.lred[3][g]);
      uint16_t* out_row = p.out + (static_cast<size_t>(sg.s) * Hq + static_cast<size_t>(sg.h) * G) * D;
      if (sg.j0 == 0 && sg.n == sg.nb) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const uint32_t two = pack2<kBf16>(acc[g] / L[g], 0.f);
          out_row[g * D + r] = static_cast<uint16_t>(two & 0xffffu);
        }
      } else {
        float* pp = p.partials + partial_slot(cta, sg.unit_first, wr) * (G * (D + 2));
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (ctid == g) {
            pp[g] = m[g];
            pp[G + g] = L[g];
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) pp[2 * G + g * D + r] = acc[g];
        __threadfence();
        finish_split_unit<kBf16, D, G>(p, sg, wr, ctid, kSoftmaxThreads, &sm.is_last,
                                       [] { named_barrier_sync(kSoftmaxBarrier, kSoftmaxThreads); });
      }
      named_barrier_sync(kSoftmaxBarrier, kSoftmaxThreads);
    }
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
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---- host side -----------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
  });
  return fn;
}

// 2-D map over a [rows][128] fp16/bf16 tensor, boxes of 64 columns x box_rows
// rows, 128-byte swizzle; rows past the end read as zero.
static bool make_map(CUtensorMap* map, const void* base, unsigned long long rows, bool bf16, uint32_t box_rows) {
  auto encode = encode_fn();
  if (encode == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool kBf16, int G>
static cudaError_t launch_tc(const Variant& v, const DecodeParams& prm, int ctas, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  const unsigned long long q_rows = static_cast<unsigned long long>(prm.num_seqs) * prm.num_q_heads;
  const unsigned long long kv_rows = static_cast<unsigned long long>(prm.num_blocks) * prm.num_kv_heads * B;
  if (kv_rows >= (1ull << 31) || q_rows >= (1ull << 31)) return cudaErrorInvalidValue;
  if (!make_map(&mq, prm.q, q_rows, kBf16, N) || !make_map(&mk, prm.k_pool, kv_rows, kBf16, B) ||
      !make_map(&mv, prm.v_pool, kv_rows, kBf16, B)) {
    return cudaErrorInvalidValue;
  }
  return launch_overlapped(pa_decode_tc_kernel<kBf16, G>, dim3(ctas), dim3(kThreads),
                           static_cast<size_t>(v.smem_bytes), stream, prm, mq, mk, mv);
}

template <bool kBf16, int G>
static Variant tc_variant() {
  return Variant{reinterpret_cast<const void*>(&pa_decode_tc_kernel<kBf16, G>), kThreads, kSmemBytes, G * (D + 2),
                 &launch_tc<kBf16, G>};
}

}  // namespace tc

bool select_tc_variant(const pa_pool_desc& pool, int group, Variant& v) {
  if (pool.head_dim != tc::D || pool.block_size != tc::B) return false;
  const bool bf16 = pool.dtype == PA_BF16;
  if (!bf16 && pool.dtype != PA_FP16) return false;
  if (group == 4) {
    v = bf16 ? tc::tc_variant<true, 4>() : tc::tc_variant<false, 4>();
    return true;
  }
  if (group == 8) {
    v = bf16 ? tc::tc_variant<true, 8>() : tc::tc_variant<false, 8>();
    return true;
  }
  return false;
}

}  // namespace pa
