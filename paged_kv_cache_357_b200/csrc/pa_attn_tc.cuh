// Paged attention on tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// What it computes (vLLM blog §"关键细节" 2; PagedAttention study notes
// ch.05 §4): softmax(scale * q K^T) V over a sequence's paged tokens, the
// normalisation merged across blocks with a running max and sum.  A unit
// pairs one kv head with R query rows, which makes both products real (if
// thin) matrix products:
//
//   S^T[token, row] = K_chunk[token, :] . Q^T[:, row]       (M=128, N=max(16,R), K=128)
//   O^T[d, row]     = V_chunk^T[d, token] . P^T[token, row] (M=128, N=max(16,2R), K=16 per step)
//
// The rows are R = G x RG: the G query heads that share the kv head (GQA),
// times RG row groups.  P^T carries 2R rows, each probability as a 16-bit
// head plus a 16-bit residual, summed in the epilogue.  Three kinds of unit
// (kMode):
//   kDecode  one sequence, RG = 1: the decode step.
//   kMulti   one sequence, RG >= q_len new query positions, position i seeing
//            the tokens up to seq_len - q_len + i (causal): speculative
//            verification and prefill chunks (CSDN "PagedAttention：分页注意力",
//            §"2026年最新进展" items 1-2).
//   kGroup   a group of up to RG sequences whose leading blocks are the same
//            physical blocks (parallel samples of one prompt, study notes
//            §6.1; prefix caching, "vLLM 是什么" §3): the unit streams the
//            shared blocks once, seen by every member's rows, then each
//            member's own blocks, seen by that member's rows only.
//
// Work partition: pa_decode_common.cuh (ranges of equal cost, 8-block chunks
// plus a fixed finish cost per unit, per CTA).  A unit split between CTAs is
// merged by the CTA that holds its first piece (see the split-unit helpers
// below).
//
// Roles (128 + 128 x WG threads, one CTA per SM):
//   warp 0      K producer: resolves block ids (32 table entries per load,
//               one batch ahead), issues 2-D TMA loads of the K tiles
//               (64-column boxes, 128-byte swizzle) into a ring of 32 KB
//               chunk stages, released when its QK is done, and a 3-D TMA
//               load of the unit's q rows.
//   warp 1      allocates TMEM; lane 0 issues QK of each chunk (tcgen05.mma,
//               tcgen05.commit) as soon as its K, q and S buffer are ready.
//   warp 2      V producer: the same walk, V tiles into their own ring
//               (one 3-D box per block, both 64-column halves), released
//               when the chunk's PV is done.  A warp issues TMA boxes one
//               lane at a time, so K and V go out in parallel.
//   warp 3      lane 0 issues PV of each chunk as soon as its P and V are
//               ready, accumulating into the O buffer of the chunk's unit
//               (units alternate between two); with QK on its own thread
//               neither product waits for the other's issue.
//   warps 4..   softmax (WG warpgroups), one TMEM lane (token row, then
//               head_dim index) per thread: read S^T from TMEM, column
//               maxima and sums by warp butterfly reduce-scatters, write P^T
//               (bf16/fp16) into a swizzled buffer, zero V rows past the
//               sequence end inside the last 16-token step.  O^T stays in
//               TMEM across a unit's chunks: it is rescaled in place only
//               when a row's reference max moves (rare past the first
//               chunk) and read once, when the unit is finished.
// The swizzled layouts written by TMA serve both products directly: the K
// tile is a K-major A operand for QK, the V tile an MN-major A operand for PV.
#pragma once

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
constexpr int kChunkTok = 128;             // tokens per chunk = MMA M of QK
constexpr int kKStages = 2;                // K is released as soon as its QK completes
constexpr int kRowBytes = 128;             // one swizzle row: 64 elements
constexpr int kHalfBytes = kChunkTok * kRowBytes;  // 64 head_dim columns x 128 tokens
constexpr int kOperandBytes = 2 * kHalfBytes;      // head_dim [0:64) then [64:128)

// Shapes that follow from the block size BB (8, 16 or 32 tokens).  A chunk
// is always 128 tokens, so CB = 16, 8 or 4 blocks.
//   V stage: [block][half][BB tokens][64 columns], one 3-D box per block
//   (both 64-column halves, kBlockBytes apart).  A 16-token PV step reads
//   two blocks (BB = 8), one block or half a block.
//   K stage, a K-major operand whose 8-token groups must sit a uniform
//   distance apart: for BB = 8 every block is one such group, so the V
//   layout serves (one 3-D box per block, groups 2 KB apart, halves 1 KB
//   apart); for BB = 16, 32 [half][128 tokens][64 columns] with two 2-D boxes
//   per block (groups 1 KB apart, halves kHalfBytes apart).
template <int BB>
struct Blk {
  static_assert(BB == 8 || BB == 16 || BB == 32, "blocks of 8, 16 or 32 tokens");
  static constexpr int CB = kChunkTok / BB;            // blocks per chunk
  static constexpr int kBlockBytes = BB * kRowBytes;   // one block's rows in one half
  static constexpr int kVBlockBytes = 2 * kBlockBytes;  // both halves of one block
  static constexpr bool kK3D = BB == 8;
  static constexpr int kKGroupBytes = kK3D ? kVBlockBytes : 8 * kRowBytes;  // K: 8-token group stride
  static constexpr int kKHalfBytes = kK3D ? kBlockBytes : kHalfBytes;       // K: second 64 columns
  static constexpr int kKBoxBytes = kK3D ? kVBlockBytes : kBlockBytes;      // K: one box (per block / half)
  static constexpr int kVGroupBytes = BB == 8 ? kVBlockBytes : 8 * kRowBytes;  // V: 8-token group stride
  // V stage offset of token t of the chunk (its row in the first half)
  __host__ __device__ static constexpr int v_offset(int t) { return (t / BB) * kVBlockBytes + (t % BB) * kRowBytes; }
};
constexpr int kWarpgroupBarrier0 = 2;       // + warpgroup index: one softmax warpgroup
constexpr int kQKWarp = 1;                 // allocates TMEM, issues QK
constexpr int kVWarp = 2;                  // the V producer (warp 0 loads q and K)
constexpr int kPVWarp = 3;                 // issues PV
constexpr int kSoftmaxWarp0 = 4;           // first softmax warp
// A row's probabilities are taken relative to a reference max that only moves
// when a score exceeds it by more than this (log2 units): p <= 2^8 stays
// exact enough in 16-bit and in the fp32 sums, and most chunks need neither
// a cross-warp max nor a rescale.
constexpr float kRescaleGap = 8.f;
// Reference max of a row that has seen no score yet: finite, so that
// score - reference is -inf for a masked score (p = 0) and never NaN, with no
// per-row test for an empty row; exp2 of it against any real score is 0.
constexpr float kNoMax = -1e30f;

enum Mode { kDecode = 0, kMulti = 1, kGroup = 2, kMultiTiled = 3 };

// kMulti: one unit per sequence (G x q_len rows fit one unit); kMultiTiled:
// several units (row tiles) per sequence, for longer q_len.  Two modes
// rather than one, so that the common single-unit form carries none of the
// tiling arithmetic.
__host__ __device__ constexpr bool is_multi(int mode) { return mode == kMulti || mode == kMultiTiled; }

// Shapes that follow from the number of query rows R of a unit.  P enters
// the PV product as two 16-bit rows per query row, p = hi + lo (the head and
// the rounding residual), so PV keeps about 16 significant bits of each
// probability instead of 8 (bf16); for R <= 8 the tail rows fill columns the
// MMA computes anyway (N = 16).
template <int R>
struct Rows {
  static_assert(R >= 1 && R <= 32 && (R & (R - 1)) == 0, "R is a power of two up to 32");
  static constexpr int Nq = R < 16 ? 16 : R;                      // MMA N of QK (q rows)
  static constexpr int Np = 2 * R < 16 ? 16 : 2 * R;              // MMA N of PV (P head + tail rows)
  static constexpr int kVStages = Np == 64 ? 3 : 4;               // V is held until its PV completes
  static constexpr int kQSlotBytes = 2 * Nq * kRowBytes;          // two 64-column halves
  // P^T is stored MN-major: one row of Np 16-bit values per token, swizzled
  // in 16-byte chunks with the pattern whose width is the row (32, 64 or 128 B)
  static constexpr int kPRowBytes = Np * 2;
  static constexpr int kPSlotBytes = kChunkTok * kPRowBytes;
  static constexpr uint32_t kPLayout = Np == 16 ? 6u : Np == 32 ? 4u : 2u;  // 32B, 64B, 128B swizzle
  // chunk index XOR for token row t (address bits [4, 4 + b) ^= bits [7, 7 + b))
  __device__ static __forceinline__ int p_swizzle(int t) {
    return Np == 16 ? ((t >> 2) & 1) : Np == 32 ? ((t >> 1) & 3) : (t & 7);
  }
  static constexpr int kColS = 0;                                 // S[0], S[1]: Nq columns each
  static constexpr int kColO = 2 * Nq;                            // O[0], O[1]: Np columns each
  static constexpr int kCols = 2 * Nq + 2 * Np;
  static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128 : 256;
  static constexpr int kPartStride = R * (D + 2);                 // floats per partial slot
  // Softmax warpgroups: one for up to 8 rows, two for 16 or 32, each taking
  // RC = R / WG of the rows (both read every token row of S and O).
  static constexpr int WG = R >= 16 ? 2 : 1;
  static constexpr int RC = R / WG;
  static constexpr int kSoftmaxThreads = 128 * WG;
  static constexpr int kThreads = 128 + kSoftmaxThreads;         // + K, QK, V and PV warps
  static constexpr int kLanesPerCol = 32 / RC;                    // lanes holding one column after a reduce
  // With two softmax warpgroups the control warpgroup hands registers to
  // them (setmaxnreg) inside the launch's allocation of 168 a thread:
  // 128 x 80 + 256 x 208 = 384 x 168 (the producers spill below 80).
  static constexpr int kCtrlRegs = 80;
  static constexpr int kSoftmaxRegs = 208;
  static constexpr int kLaunchRegs = 168;
  static_assert(WG == 1 || 128 * kCtrlRegs + kSoftmaxThreads * kSoftmaxRegs <= kThreads * kLaunchRegs,
                "the register split fits the launch's allocation");
};

template <int R>
struct TcSmem {
  using S = Rows<R>;
  uint8_t kbuf[kKStages][kOperandBytes];  // 1024-aligned regions
  uint8_t vbuf[S::kVStages][kOperandBytes];
  uint8_t q[2][S::kQSlotBytes];
  uint8_t p[2][S::kPSlotBytes];
  // a finished unit's outputs, [row][head_dim] 16-bit, written to global
  // memory by bulk copies (each warpgroup's rows by its leader)
  alignas(128) uint8_t ostage[R * D * 2];
  alignas(16) float red[2][4][R];  // per-warp column maxima, double-buffered by chunk
  // the reference max and per-warp row sums of a segment being finished,
  // by the parity of its O buffer (a segment's stash is read while the
  // next segment's may be written)
  alignas(16) float mfin[2][R];
  alignas(16) float lred[2][4][R];
  uint64_t kfull[kKStages];
  uint64_t kempty[kKStages];
  uint64_t vfull[S::kVStages];
  uint64_t vempty[S::kVStages];
  uint64_t qfull[2];
  uint64_t qempty[2];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done;                // one phase per chunk: its PV has completed
  uint64_t o_free[2];              // a segment's O buffer has been read by its finish
  uint64_t mma_done[2];            // the QK and the PV issuer's last MMAs
  RangeSmem range;
  uint32_t tmem_base;
  int abort;
  int merge_ok[2];                 // per softmax warpgroup: every other piece of the unit arrived
  int k_issued;
  int k_consumed;
  int v_issued;
  int v_consumed;
  int q_issued;
  int q_consumed;
  uint32_t sync_gen;               // generation of the new-token barrier seen before arriving
};

template <int R>
constexpr int smem_bytes() {
  return static_cast<int>(sizeof(TcSmem<R>)) + 1024;  // + alignment slack
}
constexpr int kMaxSmemPerCta = 227 * 1024;

// ---- tcgen05 / TMA primitives ------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
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

// 16 consecutive 32-bit columns of this thread's TMEM lane (completion is
// waited for separately, so several loads can be in flight).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Columns [0, NC) of this thread's TMEM lane from r (NC = 8 or a multiple of 16).
template <int NC>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t* r) {
  if constexpr (NC == 8) {
    tmem_st8(taddr, r);
  } else {
    static_assert(NC % 16 == 0, "8 or a multiple of 16 columns");
#pragma unroll
    for (int c = 0; c < NC; c += 16) tmem_st16(taddr + c, r + c);
  }
}

// Columns [0, NC) of this thread's TMEM lane (NC = 8 or a multiple of 16),
// issued without waiting; tmem_wait_ld() completes them.
template <int NC>
__device__ __forceinline__ void tmem_ld_nowait(uint32_t taddr, uint32_t* r) {
  if constexpr (NC == 8) {
    tmem_ld8_nowait(taddr, r);
  } else {
    static_assert(NC % 16 == 0, "8 or a multiple of 16 columns");
#pragma unroll
    for (int c = 0; c < NC; c += 16) tmem_ld16_nowait(taddr + c, r + c);
  }
}

template <int NC>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float* v) {
  uint32_t r[NC];
  tmem_ld_nowait<NC>(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < NC; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, sm_100 version 1, swizzle layout code
// `layout` (2 = 128 B, 4 = 64 B, 6 = 32 B).  lbo/sbo in bytes: lbo = distance
// between swizzle-atom-wide column groups of an MN-major operand (unused for
// K-major, and when the operand is one atom wide), sbo = distance between
// 8-row groups.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) |
         (static_cast<uint64_t>(layout & 7u) << 61);
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return smem_desc(saddr, lbo, sbo, 2u);
}

// Instruction descriptor of kind::f16: fp32 accumulate, A/B both bf16 or both
// fp16, each K-major or MN-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t make_idesc(bool bf16, bool a_mn_major, bool b_mn_major, int n) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(128 >> 4) << 24);
}

// Reduce R values per lane over the warp by a butterfly reduce-scatter:
// afterwards lane l holds, for column l / (32 / R), the max (kMax) or sum of
// that column over all 32 lanes.  R - 1 + log2(32 / R) shuffles in all,
// instead of 5 per column.
template <int R, bool kMax>
__device__ __forceinline__ float warp_column_reduce(float (&v)[R], int lane) {
#pragma unroll
  for (int half = R / 2, o = 16; half >= 1; half /= 2, o /= 2) {
    const bool upper = (lane & o) != 0;  // keeps columns [half, 2 half) of what it holds
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float send = upper ? v[k] : v[k + half];
      const float keep = upper ? v[k + half] : v[k];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[k] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = 16 / R; o >= 1; o /= 2) {
    const float got = __shfl_xor_sync(0xffffffffu, r, o);
    r = kMax ? fmaxf(r, got) : r + got;
  }
  return r;
}

// R consecutive floats of shared memory (16-byte aligned when R >= 4) into registers.
template <int R>
__device__ __forceinline__ void ld_row(const float* src, float (&dst)[R]) {
  if constexpr (R % 4 == 0) {
#pragma unroll
    for (int k = 0; k < R / 4; ++k) {
      const float4 v = reinterpret_cast<const float4*>(src)[k];
      dst[4 * k] = v.x;
      dst[4 * k + 1] = v.y;
      dst[4 * k + 2] = v.z;
      dst[4 * k + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < R; ++k) dst[k] = src[k];
  }
}

// One chunk of a unit: up to CB consecutive blocks of one table row, and the
// query rows that see its tokens.
struct ChunkSrc {
  int seq;             // table row
  int j;               // first logical block
  int nblk;            // blocks
  int ntok;            // valid tokens
  int len;             // tokens of the row's sequence (the causal limit's reference)
  int row_lo, row_hi;  // query rows [row_lo, row_hi) that see these tokens
  int pos0;            // multi-query: position of the unit's first row group
};

// ---- what a unit covers --------------------------------------------------------

// Token counts of the members of group g = sequences [s0, s1), at most RG
// of them, loaded together (0 past s1), and the group's shared blocks: its
// prefix length, or 0 when the group shares none.  The prefix must be
// shorter than every member's block count, so that every member keeps at
// least one block (its newest token) of its own.
template <int RG, int BB>
__device__ __forceinline__ int group_members(const DecodeParams& p, int g, int s0, int s1, int (&len)[RG]) {
  const int pb = __ldg(p.group_prefix + g);
#pragma unroll
  for (int m = 0; m < RG; ++m) len[m] = s0 + m < s1 ? checked_len(p, s0 + m, BB) : 0;
  bool fits = pb > 0;
#pragma unroll
  for (int m = 0; m < RG; ++m) fits = fits && (s0 + m >= s1 || pb < (len[m] + BB - 1) / BB);
  return fits ? pb : 0;
}

__device__ __forceinline__ bool group_ok(const DecodeParams& p, int s0, int s1, int max_members) {
  return s0 >= 0 && s1 <= p.num_seqs && s1 - s0 >= 1 && s1 - s0 <= max_members;
}

template <int kMode, int RG>
struct Source;

// A sequence: all its blocks.
template <int RG>
struct Source<kDecode, RG> {
  template <int BB>
  __device__ __forceinline__ SeqSpan span(const DecodeParams& p, int s) const {
    const int len = checked_len(p, s, BB);
    return SeqSpan{0, (len + BB - 1) / BB, len};
  }
  __device__ __forceinline__ int count(const DecodeParams& p) const { return p.num_seqs; }
  __device__ __forceinline__ int table_row(const DecodeParams&, int s) const { return s; }
  __device__ __forceinline__ int row_group0(const DecodeParams&, int s) const { return s; }
  __device__ __forceinline__ int row_groups(const DecodeParams&, int) const { return 1; }
};

// A sequence with q_len query positions, causal among the new tokens, in
// one unit.  A sequence shorter than q_len is treated as empty.
template <int RG>
struct Source<kMulti, RG> {
  template <int BB>
  __device__ __forceinline__ SeqSpan span(const DecodeParams& p, int s) const {
    int len = checked_len(p, s, BB);
    if (len < p.q_len) len = 0;
    return SeqSpan{0, (len + BB - 1) / BB, len};
  }
  __device__ __forceinline__ int count(const DecodeParams& p) const { return p.num_seqs; }
  __device__ __forceinline__ int table_row(const DecodeParams&, int s) const { return s; }
  __device__ __forceinline__ int pos0(const DecodeParams&, int) const { return 0; }
  __device__ __forceinline__ int row_group0(const DecodeParams& p, int s) const { return s * p.q_len; }
  __device__ __forceinline__ int row_groups(const DecodeParams& p, int) const { return p.q_len; }
};

// The same over several units per sequence.  Unit u is row tile t = u %
// q_tiles of sequence s = u / q_tiles: positions [t RG, min(q_len, (t + 1)
// RG)), so a sequence with G x q_len query rows past what one unit holds is
// covered by several units.  A tile reads only the blocks its last position
// sees.  A sequence shorter than q_len is treated as empty.
template <int RG>
struct Source<kMultiTiled, RG> {
  template <int BB>
  __device__ __forceinline__ SeqSpan span(const DecodeParams& p, int u) const {
    const int s = u / p.q_tiles;
    int len = checked_len(p, s, BB);
    if (len < p.q_len) len = 0;
    const int end = min(p.q_len, (u - s * p.q_tiles + 1) * RG);  // positions up to the tile's end
    const int seen = len > 0 ? len - p.q_len + end : 0;           // tokens the tile's last position sees
    return SeqSpan{0, (seen + BB - 1) / BB, len};
  }
  __device__ __forceinline__ int count(const DecodeParams& p) const { return p.num_seqs * p.q_tiles; }
  __device__ __forceinline__ int table_row(const DecodeParams& p, int u) const { return u / p.q_tiles; }
  __device__ __forceinline__ int pos0(const DecodeParams& p, int u) const { return (u % p.q_tiles) * RG; }
  __device__ __forceinline__ int row_group0(const DecodeParams& p, int u) const {
    return table_row(p, u) * p.q_len + pos0(p, u);
  }
  __device__ __forceinline__ int row_groups(const DecodeParams& p, int u) const {
    return min(RG, p.q_len - pos0(p, u));
  }
};

// A group of sequences [starts[g], starts[g+1]): the shared prefix, then each
// member's own blocks, each part starting a new granule.  On the work line a
// group unit is a run of "virtual" blocks, CB per granule; GroupWalk maps
// them back to table rows.  A group with more than RG members, or outside
// the batch, covers nothing (and is reported by group_bookkeeping).
template <int RG>
struct Source<kGroup, RG> {
  template <int BB>
  __device__ __forceinline__ SeqSpan span(const DecodeParams& p, int g) const {
    const int s0 = __ldg(p.group_starts + g), s1 = __ldg(p.group_starts + g + 1);
    if (!group_ok(p, s0, s1, RG)) return SeqSpan{0, 0, 0};
    int len[RG];
    const int pb = group_members<RG, BB>(p, g, s0, s1, len);
    constexpr int CB = Blk<BB>::CB;
    int ng = (pb + CB - 1) / CB;
#pragma unroll
    for (int m = 0; m < RG; ++m) {
      if (s0 + m < s1) ng += ((len[m] + BB - 1) / BB - pb + CB - 1) / CB;
    }
    return SeqSpan{0, ng * CB, ng * CB * BB};
  }
  __device__ __forceinline__ int count(const DecodeParams& p) const { return p.num_groups; }
  __device__ __forceinline__ int table_row(const DecodeParams& p, int g) const { return __ldg(p.group_starts + g); }
  __device__ __forceinline__ int row_group0(const DecodeParams& p, int g) const { return __ldg(p.group_starts + g); }
  __device__ __forceinline__ int row_groups(const DecodeParams& p, int g) const {
    return __ldg(p.group_starts + g + 1) - __ldg(p.group_starts + g);
  }
};

// The chunks of one segment, in order, for any kind of unit.  A sequence
// unit's chunks are consecutive blocks of its row, seen by all its rows.  A
// group unit's chunks are the shared prefix (through the first member's row,
// seen by every member's rows) and then each member's own blocks (its row,
// seen by its own G rows); the members' lengths are read once, at start.
template <int kMode, int G, int RG, int B>
struct ChunkWalk {
  static constexpr int CB = Blk<B>::CB;
  // current part: table row, next block, end block, sequence tokens, rows
  int seq, j, jend, len, row_lo, row_hi;
  int pos0;  // multi-query: position of the unit's first row group
  // group units only
  int s0, s1, pb, member;  // member = -1 while in the prefix
  int mlen[kMode == kGroup ? RG : 1];

  __device__ __forceinline__ void start(const DecodeParams& p, const Seg& sg, int rows) {
    pos0 = 0;
    if constexpr (kMode != kGroup) {
      seq = kMode == kMultiTiled ? sg.s / p.q_tiles : sg.s;
      j = sg.j0;
      jend = sg.j0 + sg.n;
      len = sg.len;
      row_lo = 0;
      row_hi = rows;
      if constexpr (kMode == kMultiTiled) pos0 = (sg.s % p.q_tiles) * RG;
    } else {
      s0 = __ldg(p.group_starts + sg.s);
      s1 = __ldg(p.group_starts + sg.s + 1);
      pb = group_members<RG, B>(p, sg.s, s0, s1, mlen);
      int skip = sg.j0 / CB;  // granules of the unit before this segment
      const int gp = (pb + CB - 1) / CB;
      if (skip < gp) {
        enter_prefix(skip);
      } else {
        skip -= gp;
        member = 0;
#pragma unroll
        for (int m = 0; m < RG; ++m) {
          const int gm = s0 + m < s1 ? ((mlen[m] + B - 1) / B - pb + CB - 1) / CB : 0;
          if (member == m && skip >= gm) {
            skip -= gm;
            member = m + 1;
          }
        }
        enter_member(skip);
      }
    }
  }

  // The chunk at the walk's position; the walk moves past it.
  __device__ __forceinline__ ChunkSrc next(const DecodeParams& p) {
    (void)p;
    ChunkSrc c;
    c.seq = seq;
    c.j = j;
    c.nblk = min(CB, jend - j);
    c.ntok = min(c.nblk * B, len - j * B);
    c.len = len;
    c.row_lo = row_lo;
    c.row_hi = row_hi;
    c.pos0 = pos0;
    j += c.nblk;
    if constexpr (kMode == kGroup) {
      if (j >= jend) {  // on to the next member with blocks of its own
        ++member;
        enter_member(0);
      }
    }
    return c;
  }

 private:
  __device__ __forceinline__ void enter_prefix(int granule) {
    member = -1;
    seq = s0;
    j = granule * CB;
    jend = pb;
    len = pb * B;
    row_lo = 0;
    row_hi = (s1 - s0) * G;
  }
  // the first member from `member` on with blocks of its own (registers only)
  __device__ __forceinline__ void enter_member(int granule) {
    int next = s1 - s0, l = 0;
#pragma unroll
    for (int m = RG - 1; m >= 0; --m) {
      if (m >= member && s0 + m < s1 && (mlen[m] + B - 1) / B > pb) {
        next = m;
        l = mlen[m];
      }
    }
    member = next;
    len = l;
    jend = (l + B - 1) / B;
    seq = s0 + member;
    j = pb + granule * CB;
    row_lo = member * G;
    row_hi = row_lo + G;
  }
};

// kGroup launches, every CTA before its own work: check that the groups
// partition the sequences and fit the kernel, and zero the outputs of groups
// with nothing to read.  Group g is handled by thread g / gridDim.x of CTA
// g % gridDim.x.
template <int RG, int B>
__device__ void group_bookkeeping(const DecodeParams& p, const Source<kGroup, RG>& src) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long g = static_cast<long long>(threadIdx.x) * gridDim.x + blockIdx.x; g < p.num_groups; g += stride) {
    const int s0 = __ldg(p.group_starts + g), s1 = __ldg(p.group_starts + g + 1);
    if (s0 < 0 || s1 < s0 || s1 > p.num_seqs || s1 - s0 > RG) {
      record_status(p.status, PA_DEV_BAD_GROUP);
      continue;
    }
    const SeqSpan sp = src.template span<B>(p, static_cast<int>(g));
    if (sp.nb > 0) continue;
    uint4* o = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(s0) * p.num_q_heads * D);
    const int n = (s1 - s0) * p.num_q_heads * D / 8;
    for (int i = 0; i < n; ++i) o[i] = make_uint4(0, 0, 0, 0);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (__ldg(p.group_starts) != 0 || __ldg(p.group_starts + p.num_groups) != p.num_seqs) {
      record_status(p.status, PA_DEV_BAD_GROUP);
    }
  }
}

// kDecode and the multi-query modes: zero the output rows of units with nothing to read
// (length 0, invalid, or shorter than q_len); unit u by CTA u % gridDim.x.
template <int kMode, int RG, int B>
__device__ void zero_empty_units(const DecodeParams& p, const Source<kMode, RG>& src) {
  const long long nctas = gridDim.x, cta = blockIdx.x;
  const int units = src.count(p);
  for (int u = threadIdx.x; u < units; u += blockDim.x) {
    if ((u % nctas) != cta) continue;
    if constexpr (is_multi(kMode)) {
      const int raw = __ldg(p.seq_lens + src.table_row(p, u));
      if (src.pos0(p, u) == 0 && raw > 0 && raw < p.q_len) record_status(p.status, PA_DEV_BAD_SEQ_LEN);
    }
    const SeqSpan sp = src.template span<B>(p, u);
    if (sp.nb > sp.first) continue;
    uint4* o = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(src.row_group0(p, u)) * p.num_q_heads * D);
    const int n = src.row_groups(p, u) * p.num_q_heads * D / 8;
    for (int i = 0; i < n; ++i) o[i] = make_uint4(0, 0, 0, 0);
    if (p.lse != nullptr) {
      float* l = p.lse + static_cast<size_t>(src.row_group0(p, u)) * p.num_q_heads;
      for (int i = 0; i < src.row_groups(p, u) * p.num_q_heads; ++i) l[i] = -INFINITY;
    }
  }
}

// ---- unit results --------------------------------------------------------------

// The output row (in units of num_q_heads x head_dim) of row group rg of
// the unit in segment sg; s0 is a group unit's first sequence.
template <int RG, int kMode>
__device__ __forceinline__ size_t out_row(const DecodeParams& p, const Seg& sg, int s0, int rg) {
  if constexpr (kMode == kMultiTiled) {
    const int s = sg.s / p.q_tiles;
    return static_cast<size_t>(s) * p.q_len + (sg.s - s * p.q_tiles) * RG + rg;
  } else if constexpr (kMode == kMulti) {
    return static_cast<size_t>(sg.s) * p.q_len + rg;
  } else if constexpr (kMode == kGroup) {
    return static_cast<size_t>(s0 + rg);
  } else {
    return static_cast<size_t>(sg.s);
  }
}

// Rows col0 .. col0 + RC - 1 of a unit, head_dim element d, from their sums
// L and unnormalised outputs a: the normalised outputs into this
// warpgroup's rows of the staging tile.  A row that saw no token (a group
// member of length 0) gets zeros.  L >= 1 whenever it is positive (the row
// max contributes 2^0), so the fast quotient keeps 22 or more bits.
template <bool kBf16, int RC>
__device__ __forceinline__ void stage_rows(uint8_t* stage, int col0, int d, const float (&L)[RC],
                                           const float (&a)[RC]) {
#pragma unroll
  for (int k = 0; k < RC; ++k) {
    const uint32_t two = pack2<kBf16>(L[k] > 0.f ? __fdividef(a[k], L[k]) : 0.f, 0.f);
    *reinterpret_cast<uint16_t*>(stage + ((col0 + k) * D + d) * 2) = static_cast<uint16_t>(two & 0xffffu);
  }
}

// By the warpgroup's leader once its rows are staged (and made visible to
// the async proxy): one bulk copy per row group of G heads (G x head_dim
// contiguous outputs), for the row groups below `rows`.
template <int G, int RG, int RC, int kMode>
__device__ __forceinline__ void issue_rows(const DecodeParams& p, const Seg& sg, int s0, int col0, int rows,
                                           const uint8_t* stage) {
  static_assert(RC % G == 0, "a warpgroup holds whole row groups");
#pragma unroll
  for (int j = 0; j < RC / G; ++j) {
    const int c = col0 + j * G;
    if (c < rows) {
      const size_t row = out_row<RG, kMode>(p, sg, s0, c / G);
      bulk_copy_s2g(p.out + (row * p.num_q_heads + static_cast<size_t>(sg.h) * G) * D, stage + c * D * 2,
                    G * D * 2);
    }
  }
  bulk_commit();
}

// Split units (study notes ch.05 §4: the online-softmax merge applied to
// the pieces of a partition).  A unit cut between CTAs is merged by the CTA
// that holds its first piece: the piece ends that CTA's range, so it is the
// last thing the CTA does, while the unit's last piece opens the range of
// the CTA after it and is long finished by then.  Every other piece
// publishes its partial state (m, l, acc per row) and counts itself in the
// unit's arrival counter, one 16-bit half per softmax warpgroup (each
// warpgroup publishes and merges its own rows); the merger waits for the
// count, merges from its own registers and the published states, and
// clears its half.  A CTA only waits for CTAs after it whose pieces of the
// unit open or fill their ranges, so no wait can close a cycle.

__device__ __forceinline__ uint32_t ld_acquire_gpu(const int32_t* ptr) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

// ---- new tokens' stores ahead of the decode (pa_decode_update and friends) ---
// The step's new-token K/V stores (vLLM blog, plain-language section) run
// inside the decode launch: every thread of every CTA takes a grid-stride
// share of the 16-byte chunks, and a grid-wide barrier closes the phase, so
// no TMA load of a block can run ahead of a store into it.  The barrier is
// two words: an arrival count and a generation number.  Each CTA reads the
// generation, then arrives; the last arrival resets the count to zero (the
// workspace is left as it was found) and advances the generation, which is
// what the waiters watch.  Every CTA of the grid arrives, with or without
// decode work; the host launches this form only when the whole grid is
// resident at once, and every wait is bounded all the same.

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// One thread per CTA, after a CTA barrier that follows the CTA's stores.
// Returns the generation to wait past.  The failure-detection test hook
// keeps CTA 0 from arriving.
__device__ __forceinline__ uint32_t grid_arrive(int32_t* slot, int test_flags) {
  __threadfence();
  fence_proxy_async_global();
  uint32_t gen;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(gen) : "l"(slot + 1) : "memory");
  if ((test_flags & kFlagTestSkipUpdateArrival) && blockIdx.x == 0) return gen;
  uint32_t prev;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(slot) : "memory");
  if (prev == gridDim.x - 1) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(slot) : "memory");
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(slot + 1) : "memory");
  }
  return gen;
}

// Bounded wait until the slot's generation moves past `gen`; afterwards the
// pools' new contents are visible to this thread's TMA loads.
__device__ __forceinline__ bool grid_wait(const int32_t* slot, uint32_t gen, const volatile int* abort_flag,
                                          unsigned long long limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (ld_acquire_gpu(slot + 1) == gen) {
    if (*abort_flag != 0 || global_timer_ns() - t0 > limit_ns) return false;
    __nanosleep(64);
  }
  fence_proxy_async_global();
  return true;
}

// New tokens: chunk i of k/v ([T][Hkv][D], D / 8 chunks a row) goes to row
// slot % B of block slot / B, same kv head.  A negative slot is a padding
// token (skipped); a slot past the pool is reported and skipped.
template <int NT, int B>
__device__ void update_write_slots(const DecodeParams& p) {
  constexpr int CPR = D / 8;
  const int Hkv = p.num_kv_heads;
  const long long total = static_cast<long long>(p.upd_num_tokens) * Hkv * CPR;
  const long long num_slots = static_cast<long long>(p.num_blocks) * B;
  const long long stride = static_cast<long long>(gridDim.x) * NT;
  uint4* kp = reinterpret_cast<uint4*>(const_cast<uint16_t*>(p.k_pool));
  uint4* vp = reinterpret_cast<uint4*>(const_cast<uint16_t*>(p.v_pool));
  for (long long i = static_cast<long long>(blockIdx.x) * NT + threadIdx.x; i < total; i += stride) {
    const int chunk = static_cast<int>(i % CPR);
    const long long th = i / CPR;  // token * Hkv + head
    const int h = static_cast<int>(th % Hkv);
    const long long slot = __ldg(p.upd_slots + th / Hkv);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (chunk == 0 && h == 0) record_status(p.status, PA_DEV_BAD_SLOT);
      continue;
    }
    const size_t dst = (static_cast<size_t>((slot / B) * Hkv + h) * B + slot % B) * CPR + chunk;
    kp[dst] = __ldg(p.upd_k + i);
    vp[dst] = __ldg(p.upd_v + i);
  }
}

// Spin (bounded by limit_ns) until bits [shift, shift + 16) of *counter
// reach `need`.
__device__ __forceinline__ bool wait_arrivals(const int32_t* counter, int shift, uint32_t need,
                                              unsigned long long limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (((ld_acquire_gpu(counter) >> shift) & 0xffffu) < need) {
    if (global_timer_ns() - t0 > limit_ns) return false;
    __nanosleep(32);
  }
  return true;
}

__device__ __forceinline__ int32_t* unit_counter(const DecodeParams& p, const Seg& sg) {
  return p.counters + static_cast<size_t>(sg.s) * p.num_kv_heads + sg.h;
}

// ---- the kernel ---------------------------------------------------------------

template <bool kBf16, int G, int RG, int kMode, int B>
__global__ void __launch_bounds__(Rows<G * RG>::kThreads, 1)
    pa_decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap map_q,
                        const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
  constexpr int R = G * RG;
  using Sh = Rows<R>;
  constexpr int Nq = Sh::Nq, Np = Sh::Np, kVStages = Sh::kVStages, kLanesPerCol = Sh::kLanesPerCol;
  constexpr int WG = Sh::WG, RC = Sh::RC, kThreads = Sh::kThreads;
  constexpr int kCtrlRegs = Sh::kCtrlRegs, kSoftmaxRegs = Sh::kSoftmaxRegs;
  constexpr int RL = RC < 8 ? 8 : RC;  // TMEM columns loaded per row set (x8 is the narrowest load used)
  static_assert(kMode != kDecode || RG == 1, "a decode unit has one row group");
  using Bk = Blk<B>;
  constexpr int CB = Bk::CB;
  using Smem = TcSmem<R>;
  const Source<kMode, RG> src;
  extern __shared__ unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long cta = blockIdx.x;
  const int Hkv = p.num_kv_heads;

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
      mbar_init(&sm.s_free[i], 4 * WG);  // one arrival per softmax warp
      mbar_init(&sm.p_full[i], 4 * WG);
      mbar_init(&sm.o_free[i], 4 * WG);
    }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.mma_done[0], 1);
    mbar_init(&sm.mma_done[1], 1);
    sm.abort = 0;
    sm.k_issued = 0;
    sm.k_consumed = 0;
    sm.v_issued = 0;
    sm.v_consumed = 0;
    sm.q_issued = 0;
    sm.q_consumed = 0;
    fence_barrier_init();
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
  }
  if (warp == kQKWarp) {
    tmem_alloc(&sm.tmem_base, Sh::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const volatile int* abort_flag = &sm.abort;
  constexpr uint32_t kColS = Sh::kColS, kColO = Sh::kColO;

  // ---- inputs may come from the previous kernel in the stream
  grid_dependency_wait();
  grid_launch_dependents();
  // The step's new tokens, stored before the partition prologue so that the
  // prologue hides the barrier; the producers wait for it before their first
  // K or V load.
  const bool upd_write = p.upd_num_tokens > 0;
  if (upd_write) {
    update_write_slots<kThreads, B>(p);
    __syncthreads();
    if (tid == 0) sm.sync_gen = grid_arrive(p.grid_sync, p.test_flags);
  }
  if constexpr (kMode == kGroup) {
    group_bookkeeping<RG, B>(p, src);
  } else {
    zero_empty_units<kMode, RG, B>(p, src);
  }
  WorkRange wr;
  Cursor cur;
  const bool has_work = decode_prologue<kThreads, B, CB>(p, sm.range, wr, cur, src);  // uniform across the CTA

  if (!has_work) {
    // nothing to stream: straight to teardown
  } else if (warp == 0 || warp == kVWarp) {
    // ===================== producers ========================================
    if constexpr (WG > 1) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    // Warp 0 loads q and K, warp 2 loads V, each walking the same chunks.  A
    // warp issues its TMA boxes one lane at a time (about 70 cycles each), so
    // one warp issuing all 32 boxes of a chunk would take longer than HBM
    // takes to deliver the chunk.
    const bool is_k = warp == 0;
    const uint64_t pol_stream = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();
    bool ok = true;
    int ci = 0, qi = 0, k_issued = 0, v_issued = 0, q_issued = 0;
    // The first K or V load waits for the stores' barrier (in this thread,
    // so that its proxy fence orders the TMA reads).
    bool gated = upd_write;
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
            // q rows: heads [h G, h G + G) of row groups [z, z + RG), one box per 64-column half
            const int z = src.row_group0(p, sg.s);
            mbar_arrive_expect_tx(&sm.qfull[qs], 2 * R * kRowBytes);
            tma_load_3d(sm.q[qs], &map_q, 0, sg.h * G, z, &sm.qfull[qs], pol_keep);
            tma_load_3d(sm.q[qs] + Nq * kRowBytes, &map_q, 64, sg.h * G, z, &sm.qfull[qs], pol_keep);
            ++q_issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ++qi;
        // K and V loads of one chunk of nblk blocks; lane l < nblk holds the
        // physical block e of the chunk's block l
        // This warp's operand of one chunk of nblk blocks; lane l < nblk holds
        // the physical block e of the chunk's block l
        auto issue = [&](int nblk, int e) -> bool {
          const int ns = is_k ? kKStages : kVStages;
          const int st = ci % ns;
          uint64_t* empty = is_k ? &sm.kempty[st] : &sm.vempty[st];
          uint64_t* full = is_k ? &sm.kfull[st] : &sm.vfull[st];
          const CUtensorMap* map = is_k ? &map_k : &map_v;
          const int y = (e * Hkv + sg.h) * B;
          bool go = true;
          if (lane == 0) {
            if (gated) {
              go = grid_wait(p.grid_sync, sm.sync_gen, abort_flag, p.wait_limit_ns);
              gated = false;
            }
            if (go) go = mbar_wait_bounded(empty, ((ci / ns) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
            if (go) mbar_arrive_expect_tx(full, nblk * Bk::kVBlockBytes);
          }
          if (!__shfl_sync(0xffffffffu, go, 0)) return false;
          if (lane < nblk) {
            if (is_k && !Bk::kK3D) {
              uint8_t* base = sm.kbuf[st] + lane * Bk::kBlockBytes;
              tma_load_2d(base, map, 0, y, full, pol_stream);
              tma_load_2d(base + kHalfBytes, map, 64, y, full, pol_stream);
            } else {
              uint8_t* buf = is_k ? sm.kbuf[st] : sm.vbuf[st];
              tma_load_3d(buf + lane * Bk::kVBlockBytes, map, 0, y, 0, full, pol_stream);
            }
          }
          __syncwarp();
          if (is_k) {
            ++k_issued;
          } else {
            ++v_issued;
          }
          ++ci;
          return true;
        };
        auto checked = [&](int e, bool used) {
          if (used && (e < 0 || e >= p.num_blocks)) {
            record_status(p.status, PA_DEV_BAD_BLOCK_ID);
            return 0;
          }
          return e;
        };
        if constexpr (kMode != kGroup) {
          // One table row: entries 32 at a time (lane l holds entry b0 + l),
          // the next batch in flight while the current one is issued.
          const int32_t* trow = p.block_tables + static_cast<size_t>(src.table_row(p, sg.s)) * p.max_nb + sg.j0;
          int e_cur = (lane < sg.n) ? __ldg(trow + lane) : 0;
          for (int b0 = 0; ok && b0 < sg.n; b0 += 32) {
            const int e_next = (b0 + 32 + lane < sg.n) ? __ldg(trow + b0 + 32 + lane) : 0;
            e_cur = checked(e_cur, b0 + lane < sg.n);
            const int b_end = min(b0 + 32, sg.n);
            for (int c0 = b0; ok && c0 < b_end; c0 += CB) {
              const int e = __shfl_sync(0xffffffffu, e_cur, (c0 - b0) + (lane & (CB - 1)));
              ok = issue(min(CB, sg.n - c0), e);
            }
            e_cur = e_next;
          }
        } else {
          // Chunks from several rows: each chunk's entries, one chunk ahead.
          ChunkWalk<kMode, G, RG, B> walk;
          walk.start(p, sg, 0);
          ChunkSrc cs = walk.next(p);
          int e_cur = (lane < cs.nblk) ? __ldg(p.block_tables + static_cast<size_t>(cs.seq) * p.max_nb + cs.j + lane) : 0;
          for (int c0 = 0; ok && c0 < sg.n; c0 += CB) {
            ChunkSrc cn = cs;
            int e_next = 0;
            if (c0 + CB < sg.n) {
              cn = walk.next(p);
              e_next = (lane < cn.nblk) ? __ldg(p.block_tables + static_cast<size_t>(cn.seq) * p.max_nb + cn.j + lane)
                                        : 0;
            }
            ok = issue(cs.nblk, checked(e_cur, lane < cs.nblk));
            cs = cn;
            e_cur = e_next;
          }
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
    if constexpr (WG > 1) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    // Lane 0 issues QK of each chunk once its K has landed, its S buffer is
    // free and its q is loaded; it sleeps in the barrier waits in between.
    if (lane == 0) {
      constexpr uint32_t kIdescQK = make_idesc(kBf16, false, false, Nq);  // K: K-major A, q: K-major B
      bool ok = true;
      int qk = 0, seg_i = 0;
      Seg sg;
      while (ok && next_seg<B, CB>(cur, sg, p, src)) {
        const int qs = seg_i & 1;
        ok = mbar_wait_bounded(&sm.qfull[qs], (seg_i >> 1) & 1, abort_flag, p.wait_limit_ns);
        const uint32_t q0 = smem_u32(sm.q[qs]);
        for (int c0 = 0; ok && c0 < sg.n; c0 += CB) {
          const int ks = qk % kKStages;
          ok = mbar_wait_bounded(&sm.kfull[ks], (qk / kKStages) & 1, abort_flag, p.wait_limit_ns) &&
               mbar_wait_bounded(&sm.s_free[qk & 1], ((qk >> 1) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k0 = smem_u32(sm.kbuf[ks]);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t a = sw128_desc(k0 + (k >> 2) * Bk::kKHalfBytes + (k & 3) * 32, 16, Bk::kKGroupBytes);
            const uint64_t b = sw128_desc(q0 + (k >> 2) * Nq * kRowBytes + (k & 3) * 32, 16, 8 * kRowBytes);
            umma(tmem + kColS + (qk & 1) * Nq, a, b, kIdescQK, k > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full[qk & 1]);
          umma_commit(&sm.kempty[ks]);
          ++qk;
        }
        if (!ok) break;
        umma_commit(&sm.qempty[qs]);  // q may be reloaded once the segment's last QK is done
        ++seg_i;
      }
      // every MMA issued above completes before TMEM is released
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
    if constexpr (WG > 1) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    // Lane 0 issues PV of each chunk once its P is written and its V has
    // landed; only the 16-token steps that hold valid tokens are issued.  A
    // segment's products accumulate in one O buffer (segments alternate
    // between two), started by its first chunk once the finish of the
    // segment before last has read that buffer.
    if (lane == 0) {
      constexpr uint32_t kIdescPV = make_idesc(kBf16, true, true, Np);  // V: MN-major A, P: MN-major B
      bool ok = true;
      int pv = 0, seg_i = 0;
      Seg sg;
      while (ok && next_seg<B, CB>(cur, sg, p, src)) {
        ChunkWalk<kMode, G, RG, B> walk;
        walk.start(p, sg, 0);
        const int ob = seg_i & 1;
        ok = mbar_wait_bounded(&sm.o_free[ob], ((seg_i >> 1) & 1) ^ 1u, abort_flag, p.wait_limit_ns);
        for (int c0 = 0; ok && c0 < sg.n; c0 += CB) {
          const int ntok = walk.next(p).ntok;
          const int pb = pv & 1;
          const int vs = pv % kVStages;
          ok = mbar_wait_bounded(&sm.p_full[pb], (pv >> 1) & 1, abort_flag, p.wait_limit_ns) &&
               mbar_wait_bounded(&sm.vfull[vs], (pv / kVStages) & 1, abort_flag, p.wait_limit_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v0 = smem_u32(sm.vbuf[vs]);
          const uint32_t p0 = smem_u32(sm.p[pb]);
          const int nks = (ntok + 15) / 16;
          for (int k = 0; k < nks; ++k) {
            const uint64_t a = sw128_desc(v0 + Bk::v_offset(16 * k), Bk::kBlockBytes, Bk::kVGroupBytes);
            // tokens [16k, 16k + 16): two groups of 8 token rows; Np fits one swizzle atom
            const uint64_t b = smem_desc(p0 + k * 16 * Sh::kPRowBytes, 0, 8 * Sh::kPRowBytes, Sh::kPLayout);
            umma(tmem + kColO + ob * Np, a, b, kIdescPV, (c0 > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&sm.pv_done);
          umma_commit(&sm.vempty[vs]);
          ++pv;
        }
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
    // ===================== softmax (warps 4..) ==============================
    if constexpr (WG > 1) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // Per chunk: the scores from TMEM, the online softmax, P^T into shared
    // memory.  The chunk's PV accumulates into its segment's O buffer in
    // TMEM, so nothing is read back per chunk: O is read once, by the
    // segment's finish, and rescaled in place on the rare chunk whose
    // reference maxima move.  The finish of a segment runs after the softmax
    // of the next segment's first chunk, so the copies and the tensor core
    // stream across unit boundaries.
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;   // token row of the chunk; head_dim index of O
    const int wg = (warp - kSoftmaxWarp0) / 4;
    const int col0 = wg * RC;         // this warpgroup's query rows: col0 .. col0 + RC - 1
    const int wg_bar = kWarpgroupBarrier0 + wg;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int my_col = col0 + lane / kLanesPerCol;  // the row this lane holds after a reduce
    const bool col_writer = (lane % kLanesPerCol) == 0;
    bool ok = true;
    int ci = 0;       // chunks started
    int pv_seen = 0;  // pv_done phases consumed: chunks whose PV has completed
    int si = 0;       // segments started
    Seg sg;
    float m_ref[RC];  // reference max of each of this warpgroup's rows (the same in all its threads)
    float l_thr[RC];  // sum of p over this thread's token rows, relative to m_ref

    // Consume the pv_done phases of every chunk before `upto`, in order (a
    // chunk's PV is only issued after its softmax, so no phase is skipped).
    auto wait_pv = [&](int upto) -> bool {
      while (pv_seen < upto) {
        const bool w = mbar_wait_bounded(&sm.pv_done, pv_seen & 1, abort_flag, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) return false;
        ++pv_seen;
      }
      tc_fence_after();
      return true;
    };

    // This warpgroup's columns of O buffer ob: the heads (col0 ..) and the
    // residuals (R + col0 ..); for R <= 8 one 16-column block holds both.
    auto o_addr = [&](int ob, int part) -> uint32_t {
      return tmem + lane_base + kColO + ob * Np + (R <= 8 ? 0 : part * R + col0);
    };
    auto load_o = [&](int ob, float (&acc)[RC]) {
      if constexpr (R <= 8) {
        uint32_t v[16];
        tmem_ld_nowait<16>(o_addr(ob, 0), v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < RC; ++k) acc[k] = __uint_as_float(v[k]) + __uint_as_float(v[R + k]);
      } else {
        uint32_t h[RC], l[RC];
        tmem_ld_nowait<RC>(o_addr(ob, 0), h);
        tmem_ld_nowait<RC>(o_addr(ob, 1), l);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < RC; ++k) acc[k] = __uint_as_float(h[k]) + __uint_as_float(l[k]);
      }
    };
    // O *= alpha per row, in place (PV of the previous chunk complete, of
    // this chunk not yet issued).
    auto rescale_o = [&](int ob, const float (&alpha)[RC]) {
      if constexpr (R <= 8) {
        uint32_t v[16];
        tmem_ld_nowait<16>(o_addr(ob, 0), v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 2 * R; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * alpha[j % R]);
        tmem_st<16>(o_addr(ob, 0), v);
      } else {
        uint32_t h[RC], l[RC];
        tmem_ld_nowait<RC>(o_addr(ob, 0), h);
        tmem_ld_nowait<RC>(o_addr(ob, 1), l);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < RC; ++k) {
          h[k] = __float_as_uint(__uint_as_float(h[k]) * alpha[k]);
          l[k] = __float_as_uint(__uint_as_float(l[k]) * alpha[k]);
        }
        tmem_st<RC>(o_addr(ob, 0), h);
        tmem_st<RC>(o_addr(ob, 1), l);
      }
      tmem_wait_st();
    };

    // Online softmax of chunk ci (the first of its segment when `first`),
    // whose PV goes to O buffer ob: P^T into the swizzled B operand.  The
    // reference maxima move only when some score exceeds them by more than
    // kRescaleGap (always on a segment's first chunk); then the chunk's row
    // maxima are reduced across the warpgroup's warps and, past the first
    // chunk, the rows of O are rescaled.  Each warpgroup decides for its own
    // rows.
    auto softmax_chunk = [&](int ci, const ChunkSrc& ch, bool first, int ob) -> bool {
      const int vs = ci % kVStages;
      const int sb = ci & 1;
      bool w = mbar_wait_bounded(&sm.s_full[sb], (ci >> 1) & 1, abort_flag, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      // whether any of this warpgroup's rows sees the chunk (a group unit's
      // member chunk is seen by that member's rows only); uniform per warpgroup
      const bool mine = kMode != kGroup || (ch.row_lo < col0 + RC && ch.row_hi > col0);
      float sN[RL];
      if (mine) {
        tmem_ld<RL>(tmem + lane_base + kColS + sb * Nq + col0, sN);
      } else {
#pragma unroll
        for (int k = 0; k < RL; ++k) sN[k] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free[sb]);

      // scores of this token row for every query row (log2 domain), masked.
      // The rows of this warpgroup that see the chunk, as a bit mask: all of
      // them unless a group unit's member chunk, and none past the chunk's
      // valid tokens.
      uint32_t vis = 0;
      if (mine && r < ch.ntok) {
        const int lo = max(ch.row_lo - col0, 0), hi = min(ch.row_hi - col0, RC);
        vis = hi > lo ? ((hi >= 32 ? 0xffffffffu : (1u << hi) - 1u) & ~((1u << lo) - 1u)) : 0u;
      }
      // causal limit: position c / G of the unit sees tokens up to lim + c / G
      const int lim = kMode == kMultiTiled ? ch.len - p.q_len + ch.pos0 - (ch.j * B + r)
                                           : ch.len - p.q_len - (ch.j * B + r);
      // d = score - reference max, one FFMA a row; the same d decides the
      // rescale and, when none is needed, feeds the exponential
      auto row_valid = [&](int k) {
        bool valid = ((vis >> k) & 1u) != 0;
        if constexpr (is_multi(kMode)) valid = valid && lim + (col0 + k) / G >= 0;  // causal
        return valid;
      };
      float d[RC];
      bool over = first;
#pragma unroll
      for (int k = 0; k < RC; ++k) {
        d[k] = row_valid(k) ? fmaf(sN[k], p.scale_log2, -m_ref[k]) : -INFINITY;
        over |= d[k] > kRescaleGap;
      }
      const bool rescale = named_barrier_or(wg_bar, 128, over);  // uniform per warpgroup
      if (rescale) {
        if (mine) {
          float v[RC];
#pragma unroll
          for (int k = 0; k < RC; ++k) v[k] = row_valid(k) ? sN[k] * p.scale_log2 : -INFINITY;  // the scores
          const float wm = warp_column_reduce<RC, true>(v, lane);
          if (col_writer) sm.red[sb][quad][my_col] = wm;
        }
        named_barrier_sync(wg_bar, 128);
        float cm[RC], tt[RC];
        if (mine) {
          ld_row<RC>(sm.red[sb][0] + col0, cm);
#pragma unroll
          for (int w2 = 1; w2 < 4; ++w2) {
            ld_row<RC>(sm.red[sb][w2] + col0, tt);
#pragma unroll
            for (int k = 0; k < RC; ++k) cm[k] = fmaxf(cm[k], tt[k]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < RC; ++k) cm[k] = -INFINITY;
        }
        float alpha[RC];
#pragma unroll
        for (int k = 0; k < RC; ++k) {
          const float m_old = first ? -INFINITY : m_ref[k];
          const float m_new = fmaxf(fmaxf(m_old, cm[k]), kNoMax);
          alpha[k] = fast_exp2(m_old - m_new);
          d[k] = row_valid(k) ? fmaf(sN[k], p.scale_log2, -m_new) : -INFINITY;  // against the new reference
          m_ref[k] = m_new;
          l_thr[k] = first ? 0.f : l_thr[k] * alpha[k];
        }
        // the rows of O rescaled in place once the previous chunk's PV has
        // completed (this chunk's PV is issued only after P is released);
        // done here so that alpha is dead before the exponentials
        if (!first) {
          if (!wait_pv(ci)) return false;
          rescale_o(ob, alpha);
        }
      }
      float pr[RC];
#pragma unroll
      for (int k = 0; k < RC; ++k) {
        pr[k] = fast_exp2(d[k]);  // 0 for a masked score
        l_thr[k] += pr[k];
      }
      // P^T, MN-major: token row r holds at position c the head of query row
      // c's probability and at R + c its rounding residual, written as whole
      // 16-byte chunks of 8 values (this warpgroup's rows col0 .. col0 + RC).
      // The buffer's last reader, PV of chunk ci - 2, completed before chunk
      // ci - 1 was released.
      const int pb = ci & 1;
      {
        uint8_t* prow = sm.p[pb] + r * Sh::kPRowBytes;
        const int swz = Sh::p_swizzle(r);
        constexpr int kW = (RC + 1) / 2;  // 32-bit words of RC 16-bit values
        uint32_t hw[kW], lw[kW];
#pragma unroll
        for (int k = 0; k < kW; ++k) {
          const float a0 = pr[2 * k], a1 = (2 * k + 1 < RC) ? pr[2 * k + 1] : 0.f;
          hw[k] = pack2<kBf16>(a0, a1);
          float h0, h1;
          unpack2<kBf16>(hw[k], h0, h1);
          lw[k] = pack2<kBf16>(a0 - h0, a1 - h1);
        }
        auto put = [&](int chunk, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
          *reinterpret_cast<uint4*>(prow + ((chunk ^ swz) << 4)) = make_uint4(w0, w1, w2, w3);
        };
        if constexpr (RC >= 8) {
#pragma unroll
          for (int j = 0; j < RC / 8; ++j) {
            put(col0 / 8 + j, hw[4 * j], hw[4 * j + 1], hw[4 * j + 2], hw[4 * j + 3]);
            put((R + col0) / 8 + j, lw[4 * j], lw[4 * j + 1], lw[4 * j + 2], lw[4 * j + 3]);
          }
        } else if constexpr (RC == 4) {  // heads 0..3, residuals 4..7
          put(0, hw[0], hw[1], lw[0], lw[1]);
        } else if constexpr (RC == 2) {  // heads 0..1, residuals 2..3
          put(0, hw[0], lw[0], 0u, 0u);
        } else {  // one row: head 0, residual 1
          put(0, (hw[0] & 0xffffu) | (lw[0] << 16), 0u, 0u, 0u);
        }
      }
      // V rows past the sequence end inside the last 16-token step are zeroed
      // so that 0 * (whatever they hold) cannot reach the output
      if (col0 == 0 && (ch.ntok & 15) != 0 && r >= ch.ntok && r < ((ch.ntok + 15) & ~15)) {
        (void)mbar_wait_bounded(&sm.vfull[vs], (ci / kVStages) & 1, abort_flag, p.wait_limit_ns);
        uint4* v0 = reinterpret_cast<uint4*>(sm.vbuf[vs] + Bk::v_offset(r));
        uint4* v1 = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(v0) + Bk::kBlockBytes);
#pragma unroll
        for (int i = 0; i < kRowBytes / 16; ++i) {
          v0[i] = make_uint4(0, 0, 0, 0);
          v1[i] = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      // the previous chunk's PV must be complete before this chunk's PV may
      // add to O (and before P's buffer comes round again)
      if (!wait_pv(ci)) return false;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[pb]);
      return true;
    };

    const bool leader = quad == 0 && lane == 0;  // this warpgroup's first thread
    // A published partial state's arrival, counted by the leader after the
    // next chunk (the release fence then finds the stores long done)
    int32_t* arrival = nullptr;
    uint32_t arrival_add = 0;
    auto count_arrival = [&]() {
      if (arrival != nullptr) {
        __threadfence();
        atomicAdd(reinterpret_cast<unsigned int*>(arrival), arrival_add);
        arrival = nullptr;
      }
    };

    // A segment's row sums and reference maxima, put aside (in stash buffer
    // sb, the parity of its O buffer) before the next segment's first
    // softmax resets them: sums reduced over the warp into lred, maxima into
    // mfin.  The warpgroup barrier of the next chunk's softmax orders them
    // before finish_segment reads them.
    auto stash_segment = [&](int sb) {
      float v[RC];
#pragma unroll
      for (int k = 0; k < RC; ++k) v[k] = l_thr[k];
      const float ls = warp_column_reduce<RC, false>(v, lane);
      if (col_writer) sm.lred[sb][quad][my_col] = ls;
      if (quad == 0 && lane < RC) {
        float m = m_ref[0];
#pragma unroll
        for (int k = 1; k < RC; ++k) m = lane == k ? m_ref[k] : m;
        sm.mfin[sb][col0 + lane] = m;
      }
    };

    // The finish of a segment whose PVs have all completed, by each
    // warpgroup for its own rows: the outputs of a whole unit; for a split
    // unit, its partial state published, or (its first piece) the merge of
    // every piece.  Its O buffer ob is read once and handed back to the PV
    // issuer.  s0 is a group unit's first sequence.
    auto finish_segment = [&](const Seg& fs, int rows, int ob, int s0) {
      float acc[RC];
      load_o(ob, acc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free[ob]);
      float L[RC];
#pragma unroll
      for (int k = 0; k < RC; ++k) {
        const int c = col0 + k;
        L[k] = (sm.lred[ob][0][c] + sm.lred[ob][1][c]) + (sm.lred[ob][2][c] + sm.lred[ob][3][c]);
      }
      const bool opens = fs.j0 == fs.first, closes = fs.j0 + fs.n == fs.nb;
      // the outputs of this warpgroup's rows through the staging tile (the
      // previous finish's copies have read it by now); with p.lse, each row's
      // log normaliser, m + log2 l in the log2 domain of the scores, as a
      // natural log, by the thread of the warpgroup's first warp whose lane
      // is the row
      auto emit = [&](const float (&Mx)[RC]) {
        if (leader) bulk_wait_read();
        named_barrier_sync(wg_bar, 128);
        stage_rows<kBf16, RC>(sm.ostage, col0, r, L, acc);
        fence_proxy_async_smem();
        named_barrier_sync(wg_bar, 128);
        if (leader) issue_rows<G, RG, RC, kMode>(p, fs, s0, col0, rows, sm.ostage);
        if constexpr (kMode != kDecode) return;  // pa_decode_lse runs the decode mode only
        if (p.lse != nullptr && quad == 0 && lane < RC && col0 + lane < rows) {
          float l = L[0], m = Mx[0];
#pragma unroll
          for (int k = 1; k < RC; ++k) {
            l = lane == k ? L[k] : l;
            m = lane == k ? Mx[k] : m;
          }
          const int c = col0 + lane;
          const size_t row = out_row<RG, kMode>(p, fs, s0, c / G);
          p.lse[row * p.num_q_heads + static_cast<size_t>(fs.h) * G + c % G] =
              l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
        }
      };
      if (opens && closes) {
        float Mw[RC];
        if constexpr (kMode == kDecode) {
          if (p.lse != nullptr) ld_row<RC>(sm.mfin[ob] + col0, Mw);
        }
        emit(Mw);
        return;
      }
      int32_t* counter = unit_counter(p, fs);
      const int shift = 16 * wg;
      if (!opens) {
        // publish: m, l of this warpgroup's rows, then acc; the arrival is
        // counted after the next chunk, once these stores have drained
        float* pp = p.partials + partial_slot(cta, fs.unit_first, wr) * Sh::kPartStride;
        if (quad == 0 && lane < RC) {
          pp[col0 + lane] = sm.mfin[ob][col0 + lane];
          pp[R + col0 + lane] = (sm.lred[ob][0][col0 + lane] + sm.lred[ob][1][col0 + lane]) +
                                (sm.lred[ob][2][col0 + lane] + sm.lred[ob][3][col0 + lane]);
        }
#pragma unroll
        for (int k = 0; k < RC; ++k) pp[2 * R + (col0 + k) * D + r] = acc[k];
        named_barrier_sync(wg_bar, 128);
        if (leader) {
          arrival = counter;
          arrival_add = 1u << shift;
        }
        return;
      }
      // merge: this CTA holds the unit's first piece; pieces first + 1 ..
      // last were published by the CTAs after it
      const long long first = cta;
      const long long last = cta_of(fs.unit_last, wr.total, wr.nparts);
      const uint32_t need = static_cast<uint32_t>(last - first);
      if (leader) {
        const bool got = wait_arrivals(counter, shift, need, p.wait_limit_ns);
        if (got) {
          atomicSub(reinterpret_cast<unsigned int*>(counter), need << shift);  // back to zero for the next launch
        } else {
          record_status(p.status, PA_DEV_TIMEOUT);
        }
        sm.merge_ok[wg] = got;
      }
      named_barrier_sync(wg_bar, 128);
      if (!sm.merge_ok[wg]) return;
      float M[RC];
      ld_row<RC>(sm.mfin[ob] + col0, M);
      for (long long cc = first + 1; cc <= last; ++cc) {
        const float* pp = p.partials + partial_slot(cc, fs.unit_first, wr) * Sh::kPartStride;
        float mp[RC], lp[RC], ap[RC];
#pragma unroll
        for (int k = 0; k < RC; ++k) {
          mp[k] = __ldcg(pp + col0 + k);
          lp[k] = __ldcg(pp + R + col0 + k);
          ap[k] = __ldcg(pp + 2 * R + (col0 + k) * D + r);
        }
#pragma unroll
        for (int k = 0; k < RC; ++k) {
          const float mn = fmaxf(M[k], mp[k]);
          const float wa = fast_exp2(M[k] - mn), wb = fast_exp2(mp[k] - mn);
          L[k] = fmaf(L[k], wa, lp[k] * wb);
          acc[k] = fmaf(acc[k], wa, ap[k] * wb);
          M[k] = mn;
        }
      }
      emit(M);
    };

#pragma unroll
    for (int k = 0; k < RC; ++k) {
      m_ref[k] = kNoMax;
      l_thr[k] = 0.f;
    }
    Seg prev;               // the segment whose finish is still due
    int prev_rows = 0, prev_s0 = 0;
    bool have_prev = false;
    while (ok && next_seg<B, CB>(cur, sg, p, src)) {
      const int rows = G * src.row_groups(p, sg.s);
      ChunkWalk<kMode, G, RG, B> walk;
      walk.start(p, sg, rows);
      const int ob = si & 1;
      for (int c0 = 0; c0 < sg.n; c0 += CB) {
        if (c0 == 0 && have_prev) stash_segment(ob ^ 1);
        ok = softmax_chunk(ci, walk.next(p), c0 == 0, ob);
        if (!ok) break;
        ++ci;
        if (leader) count_arrival();
        if (c0 == 0 && have_prev) {  // every PV of the previous segment is complete
          finish_segment(prev, prev_rows, ob ^ 1, prev_s0);
          have_prev = false;
        }
      }
      if (!ok) break;
      prev = sg;
      prev_rows = rows;
      if constexpr (kMode == kGroup) prev_s0 = walk.s0;
      have_prev = true;
      ++si;
    }
    if (ok && have_prev) {
      ok = wait_pv(ci);
      if (ok) {
        const int ob = (si - 1) & 1;
        stash_segment(ob);
        named_barrier_sync(wg_bar, 128);
        finish_segment(prev, prev_rows, ob, prev_s0);
      }
    }
    if (leader) {
      count_arrival();
      bulk_wait_read();  // the staging tile stays until its copies have read it
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
  if (warp == kQKWarp) tmem_dealloc(tmem, Sh::kTmemCols);
}

// ---- host side -----------------------------------------------------------------

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Tensor map over a packed fp16/bf16 tensor whose innermost dimension is
// head_dim (128) and whose outer dimensions are outer[0..rank-2], innermost
// first; boxes of 64 columns x outer_box, 128-byte swizzle; coordinates past
// the end read as zero.
inline bool make_map(CUtensorMap* map, const void* base, int rank, const unsigned long long* outer,
                     const uint32_t* outer_box, bool bf16) {
  auto encode = encode_fn();
  if (encode == nullptr || rank < 2 || rank > 3) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), 1, 1};
  cuuint64_t strides[2] = {0, 0};
  cuuint32_t box[3] = {64, 1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  cuuint64_t stride = static_cast<cuuint64_t>(D) * 2;
  for (int i = 1; i < rank; ++i) {
    dims[i] = outer[i - 1];
    box[i] = outer_box[i - 1];
    strides[i - 1] = stride;
    stride *= outer[i - 1];
  }
  const CUresult r = encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                            static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A pool as a 3-D tensor (64 columns, rows, 2 halves 128 bytes apart): one
// box of 64 x block x 2 lands a block's rows as [half][block][64] in shared
// memory.
inline bool make_map_halves(CUtensorMap* map, const void* base, unsigned long long rows, int block, bool bf16) {
  auto encode = encode_fn();
  if (encode == nullptr) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), 2};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(block), 2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The three tensor maps of a launch, kept for the launches that follow: a
// map depends only on the kernel instance (box shapes, element type), the
// operand addresses and the extents, which make the key, so a cached map is
// the one a fresh encode would give.  A loop that decodes into the same
// buffers encodes its maps once.
struct LaunchMaps {
  const void* kernel;
  const void *q, *k, *v;
  unsigned long long q_rows, kv_rows;
  int num_q_heads;
  CUtensorMap mq, mk, mv;
};

inline bool cached_maps(const LaunchMaps& want, CUtensorMap& mq, CUtensorMap& mk, CUtensorMap& mv,
                        bool (*encode)(const LaunchMaps&, CUtensorMap&, CUtensorMap&, CUtensorMap&)) {
  constexpr int kEntries = 16;
  static std::mutex mu;
  static LaunchMaps cache[kEntries];
  static int n_used = 0, next = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_used; ++i) {
      const LaunchMaps& e = cache[i];
      if (e.kernel == want.kernel && e.q == want.q && e.k == want.k && e.v == want.v && e.q_rows == want.q_rows &&
          e.kv_rows == want.kv_rows && e.num_q_heads == want.num_q_heads) {
        mq = e.mq;
        mk = e.mk;
        mv = e.mv;
        return true;
      }
    }
  }
  if (!encode(want, mq, mk, mv)) return false;
  std::lock_guard<std::mutex> lock(mu);
  LaunchMaps& slot = cache[next];
  slot = want;
  slot.mq = mq;
  slot.mk = mk;
  slot.mv = mv;
  next = (next + 1) % kEntries;
  if (n_used < kEntries) ++n_used;
  return true;
}

template <bool kBf16, int G, int RG, int B>
bool encode_launch_maps(const LaunchMaps& w, CUtensorMap& mq, CUtensorMap& mk, CUtensorMap& mv) {
  const unsigned long long q_outer[2] = {static_cast<unsigned long long>(w.num_q_heads), w.q_rows};
  const uint32_t q_box[2] = {static_cast<uint32_t>(G), static_cast<uint32_t>(RG)};
  const unsigned long long kv_outer[1] = {w.kv_rows};
  const uint32_t kv_box[1] = {static_cast<uint32_t>(B)};
  const bool k_ok = Blk<B>::kK3D ? make_map_halves(&mk, w.k, w.kv_rows, B, kBf16)
                                 : make_map(&mk, w.k, 2, kv_outer, kv_box, kBf16);
  return k_ok && make_map(&mq, w.q, 3, q_outer, q_box, kBf16) && make_map_halves(&mv, w.v, w.kv_rows, B, kBf16);
}

template <bool kBf16, int G, int RG, int kMode, int B>
cudaError_t launch_tc(const Variant& v, const DecodeParams& prm, int ctas, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  const unsigned long long q_rows =
      static_cast<unsigned long long>(prm.num_seqs) * (is_multi(kMode) ? prm.q_len : 1);
  const unsigned long long kv_rows = static_cast<unsigned long long>(prm.num_blocks) * prm.num_kv_heads * B;
  if (kv_rows >= (1ull << 31) || q_rows >= (1ull << 31)) return cudaErrorInvalidValue;
  LaunchMaps want{};
  want.kernel = reinterpret_cast<const void*>(&pa_decode_tc_kernel<kBf16, G, RG, kMode, B>);
  want.q = prm.q;
  want.k = prm.k_pool;
  want.v = prm.v_pool;
  want.q_rows = q_rows;
  want.kv_rows = kv_rows;
  want.num_q_heads = prm.num_q_heads;
  if (!cached_maps(want, mq, mk, mv, &encode_launch_maps<kBf16, G, RG, B>)) return cudaErrorInvalidValue;
  if constexpr (Rows<G * RG>::WG > 1) {
    // setmaxnreg only moves registers inside the launch's allocation; should
    // a build give the kernel fewer than the split needs, the softmax warps'
    // increase would wait forever, so such a kernel is not launched.
    static const bool regs_fit = [] {
      cudaFuncAttributes a{};
      return cudaFuncGetAttributes(&a, pa_decode_tc_kernel<kBf16, G, RG, kMode, B>) == cudaSuccess &&
             a.numRegs * Rows<G * RG>::kThreads >=
                 128 * Rows<G * RG>::kCtrlRegs + Rows<G * RG>::kSoftmaxThreads * Rows<G * RG>::kSoftmaxRegs;
    }();
    if (!regs_fit) return cudaErrorInvalidConfiguration;
  }
  return launch_overlapped(pa_decode_tc_kernel<kBf16, G, RG, kMode, B>, dim3(ctas), dim3(Rows<G * RG>::kThreads),
                           static_cast<size_t>(v.smem_bytes), stream, prm, mq, mk, mv);
}

// Partition cost of finishing a unit, in 1/8 granules: what the finish (row
// sums, outputs or partial state, the merge) adds to a CTA's time beyond
// what the pipeline hides; it grows with the rows a unit carries.  Values
// from sweeps on B200 (Llama-3-8B decode: 2 to 3 best; q_len 4 multi-query
// at 16 rows: 6; shared-prefix group units: 20, 0.8 % ahead of 10 and 32).
constexpr int unit_finish_cost(int kMode, int R) {
  return kMode == kDecode ? (R <= 4 ? 2 : 4) : kMode == kGroup ? 20 : (R <= 8 ? 4 : R <= 16 ? 6 : 10);
}

template <bool kBf16, int G, int RG, int kMode, int B = 16>
Variant tc_variant() {
  constexpr int R = G * RG;
  static_assert(smem_bytes<R>() <= kMaxSmemPerCta, "shared memory of one CTA");
  return Variant{reinterpret_cast<const void*>(&pa_decode_tc_kernel<kBf16, G, RG, kMode, B>), Rows<R>::kThreads,
                 smem_bytes<R>(), Rows<R>::kPartStride, &launch_tc<kBf16, G, RG, kMode, B>,
                 unit_finish_cost(kMode, R), true};
}

// head_dim 128, a 16-bit pool, and a block size the instances cover: 8, 16
// or 32 tokens for the decode (any_block), 16 for the other modes.
inline bool tc_pool_ok(const pa_pool_desc& pool, bool any_block = false) {
  const bool block_ok = pool.block_size == 16 || (any_block && (pool.block_size == 8 || pool.block_size == 32));
  return pool.head_dim == D && block_ok && (pool.dtype == PA_BF16 || pool.dtype == PA_FP16);
}

// Row groups per unit for q_len positions of G heads: the smallest power of
// two >= q_len while G times that fits 32 rows (one unit per sequence),
// else 32 / G (several units, row tiles, per sequence); 0 for G outside
// 1..32.
inline int row_groups_for(int G, int q_len) {
  if (G <= 0 || G > 32 || q_len <= 0) return 0;
  int r = 1;
  while (r < q_len && G * r < 32) r *= 2;
  return r;
}

// Row tiles (units) per sequence for q_len positions at rg row groups a unit.
inline int row_tiles_for(int q_len, int rg) { return rg > 0 ? (q_len + rg - 1) / rg : 0; }

// The multi-query instances at blocks of B tokens: one unit per sequence for
// G x RG <= 32 rows (RG a power of two), row tiles of 32 rows beyond.
template <bool kBf16, int B>
bool pick_multi(int G, int RG, bool tiled, Variant& v) {
#define PA_MULTI_CASE(g, rg)                         \
  if (G == g && RG == rg && !tiled) {                \
    v = tc_variant<kBf16, g, rg, kMulti, B>();       \
    return true;                                     \
  }
  PA_MULTI_CASE(1, 2) PA_MULTI_CASE(1, 4) PA_MULTI_CASE(1, 8) PA_MULTI_CASE(1, 16) PA_MULTI_CASE(1, 32)
  PA_MULTI_CASE(2, 2) PA_MULTI_CASE(2, 4) PA_MULTI_CASE(2, 8) PA_MULTI_CASE(2, 16)
  PA_MULTI_CASE(4, 2) PA_MULTI_CASE(4, 4) PA_MULTI_CASE(4, 8)
  PA_MULTI_CASE(8, 2) PA_MULTI_CASE(8, 4)
#undef PA_MULTI_CASE
#define PA_TILED_CASE(g, rg)                         \
  if (G == g && RG == rg && tiled) {                 \
    v = tc_variant<kBf16, g, rg, kMultiTiled, B>();  \
    return true;                                     \
  }
  PA_TILED_CASE(1, 32) PA_TILED_CASE(2, 16) PA_TILED_CASE(4, 8) PA_TILED_CASE(8, 4)
#undef PA_TILED_CASE
  return false;
}

}  // namespace tc
}  // namespace pa
