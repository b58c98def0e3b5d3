// fp8_mm: scaled FP8 GEMM (NT, batched with stride-0 broadcast) for sm_100a.
//
// Computes Y[b,m,n] = bf16(sum_k A[b,m,k] B[b,n,k] * sinv_a * sinv_b + bias[n])
// as the AstrAI pages describe it ("tests/extension": bias-fusion commit --
// the fp32 bias is added before the single bf16 rounding, guarded N tails,
// batch broadcast of the bias; 3D batched commit -- batch strides, size-1
// batches broadcast at stride 0; grouped rasterisation keeps the shared
// operand stripe hot in L2).
//
// B200 design (the pages' kernels are sm_89 register-fragment MMAs; none of
// that carries over):
//   * persistent kernel, one CTA per SM, 10 warps with fixed roles:
//       warp 0      TMA producer: 128x128-byte A and BNx128-byte B tiles,
//                   128B-swizzled, into a STAGES-deep shared-memory ring
//                   guarded by full/empty mbarriers;
//       warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//                   (kind::f8f6f4, M=128, N=BN, K=32 per instruction), fp32
//                   accumulators in TMEM, double-buffered (2 x BN columns) so
//                   the epilogue of tile i overlaps the mainloop of tile i+1;
//       warps 2..9  epilogue: two warps per TMEM lane quadrant, each on half
//                   the columns; tcgen05.ld 2x32 columns per wait, one fmaf
//                   per element (acc * sinv_a*sinv_b + bias), one bf16
//                   rounding, 32x32 TMA stores from swizzled staging buffers
//                   (guarded plain stores when output rows are unaligned).
//   * every mbarrier wait is bounded by a %globaltimer budget; a wait that
//     runs out records the site in the library error word, raises a shared
//     abort flag so the other roles leave their loops, waits (bounded) for
//     the copies and MMAs it issued, frees TMEM and returns.
//   * no TMA multicast anywhere: the kernel stays legal when several GPUs
//     run replicas.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "fp8_ring.cuh"

namespace fp8ds {
namespace {

constexpr int kBM = 128;      // rows of A per tile (UMMA M)
constexpr int kBK = 128;      // K bytes (= fp8 elements) per stage: one 128B swizzle atom row
constexpr int kUmmaK = 32;    // K per tcgen05.mma for 8-bit operands
constexpr int kEpiWarps = 8;      // two warps per TMEM lane quadrant, each owning half the columns
constexpr int kThreadsMM = 32 * (2 + kEpiWarps);
constexpr int kStagingBytes = 2048;  // one 32x32 bf16 box per staging buffer

// PAIR = 1: one CTA computes a 128 x BN tile.  PAIR = 2: a cluster of two
// CTAs on two SMs computes a 256 x BN tile with tcgen05 cta_group::2; each CTA
// holds 128 rows of A, BN/2 rows of B and its 128 x BN half of the accumulator.
template <int BN, int PAIR>
struct Cfg {
  static constexpr int kBRows = BN / PAIR;
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = kBRows * kBK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024) / kStageBytes;
  static constexpr int kTmemCols = 2 * BN;  // two accumulators
  static constexpr int kStagingOffset = kStages * kStageBytes;  // 2 buffers per epilogue warp
  static constexpr int kBarOffset = kStagingOffset + kEpiWarps * 2 * kStagingBytes;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // + barriers + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert((2 * kStages + 5) * 8 + 16 + 4 * kEpiWarps + 8 <= 256,
                "barrier area: barriers, TMEM slot, abort, amax, stall barrier");
};

struct MmParams {
  int M, N, K;
  int m_tiles, n_tiles, k_blocks, tiles_per_batch, tiles_total, group_m;
  int a_bcast, b_bcast;
  int a_mn, b_mn;    // operand stored MN-major ([K][M] / [K][N], M or N contiguous)
  // Work split (data-parallel + stream-K).  Tiles [0, dp_tiles) are whole
  // tiles, dealt round-robin to the grid's CTAs (pairs).  The k-block
  // iterations of the remaining tiles, numbered g = (t - dp_tiles) * k_blocks
  // + kb, form one range [0, sk_iters) cut into sk_ctas contiguous pieces;
  // piece s = [s*sk_iters/sk_ctas, (s+1)*sk_iters/sk_ctas) runs on CTA s
  // after its whole tiles.  A piece that starts inside a tile writes its
  // float32 partial to slot s of `ws` and counts up flags[s]; the CTA holding
  // the tile's k-block 0 waits for those flags, adds the partials of the
  // following pieces in piece order and stores the tile.
  int dp_tiles, sk_ctas;
  int64_t sk_iters;
  float* ws;
  uint32_t* flags;
  int64_t c_stride;  // elements between output batches
  const float* sinv_a;
  const float* sinv_b;
  const float* bias;
  uint16_t* out;
  int out_vec;       // 16-byte stores are legal for full 8-column groups
  int tma_store;     // output leaves through TMA stores (tmC valid)
  int bias_vec;      // bias is 16-byte aligned
  uint32_t idesc;
  uint32_t* err;
  unsigned long long wait_ns;  // budget of the waits on another role's progress
  uint32_t stall;              // wait site that waits on a never-completed barrier (testing), else 0
  // Epilogue variants (kernel template EPI): an FP8 bias, dequantised as
  // fp32(code * *bias_scale), and FP8 output codes of fp32(y * *r_scale) with
  // max |y| folded into the output's ring by the CTA that finishes last.
  const uint8_t* bias8;
  const float* bias_scale;
  int bias_fmt;
  int out_fmt;
  uint8_t* out8;
  int out8_vec;      // code rows are 16-byte aligned: codes leave through TMA stores
  float* r_history;
  int32_t* r_idx;
  float* r_scale;
  float* r_scale_inv;
  uint32_t* r_scratch;  // [0] amax bits, [1] CTA ticket; zero between calls
  float* amax_out;      // data-parallel shard: the amax goes here, no fold
};

constexpr int kEpiOut8 = 1;   // EPI bit: FP8 output codes + output ring fold
constexpr int kEpiBias8 = 2;  // EPI bit: FP8 bias codes

// Value of one FP8 code (exact in fp32; NaN codes give NaN).
__device__ __forceinline__ float fp8_value(uint8_t c, int fmt) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(c, fmt == FP8_E5M2 ? __NV_E5M2 : __NV_E4M3);
  return __half2float(__half(h));
}

// Dequantised FP8 bias of columns n .. n+3, 0 beyond N.
__device__ __forceinline__ float4 bias8_4(const MmParams& p, int n, float bsc) {
  float e[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) e[q] = n + q < p.N ? __fmul_rn(fp8_value(__ldg(p.bias8 + n + q), p.bias_fmt), bsc) : 0.f;
  return make_float4(e[0], e[1], e[2], e[3]);
}

// FP8 output: this CTA's max |y| (per epilogue warp in amax_s) joins the
// ring's scratch word; the CTA that draws the last of gridDim.x tickets takes
// the grid's amax, clears the scratch words and commits the ring.  ring_s
// holds the ring's history, idx and scale as read at launch (only this fold
// writes them).  Run by one thread after the CTA's epilogue.
__device__ __noinline__ void out8_ticket_fold(const MmParams& p, const float* amax_s, const float* ring_s) {
  float m = 0.0f;
#pragma unroll
  for (int w = 0; w < kEpiWarps; ++w) m = fmaxf(m, amax_s[w]);
  // The CTA's amax goes in with an atom.max whose return value the ticket's
  // address depends on (bit 31 of a non-negative float: 0 at run time,
  // opaque to the compiler), so the ticket is issued only once the amax is
  // in L2; the CTA with the last ticket exchanges the word only after that
  // ticket returned, i.e. after every CTA's amax was performed there.  No
  // fence: a release-ordered ticket would wait for the CTA's output stores.
  uint32_t old, dep, t;
  asm volatile("atom.relaxed.gpu.global.max.u32 %0, [%1], %2;" : "=r"(old) : "l"(p.r_scratch), "r"(__float_as_uint(m))
               : "memory");
  asm volatile("shr.u32 %0, %1, 31;" : "=r"(dep) : "r"(old));
  asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], 1;" : "=r"(t) : "l"(p.r_scratch + 1 + dep) : "memory");
  if (t != gridDim.x - 1) return;
  uint32_t bits;
  asm volatile("atom.relaxed.gpu.global.exch.b32 %0, [%1], 0;" : "=r"(bits) : "l"(p.r_scratch) : "memory");
  asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(p.r_scratch + 1) : "memory");
  float hist[kHistoryLen];
#pragma unroll
  for (int i = 0; i < kHistoryLen; ++i) hist[i] = ring_s[i];
  const int idx = __float_as_int(ring_s[kHistoryLen]);
  const float s_used = ring_s[kHistoryLen + 1];
  const float a = __uint_as_float(bits);
  if (p.amax_out != nullptr) {  // shard of a data-parallel output: the fold follows a cross-rank MAX
    *p.amax_out = a;
    *p.r_scale_inv = __frcp_rn(s_used);
    return;
  }
  if (p.out_fmt == FP8_E5M2)
    ring_commit<FP8_E5M2>(a, hist, idx, p.r_history, p.r_idx, p.r_scale, p.r_scale_inv, s_used);
  else
    ring_commit<FP8_E4M3>(a, hist, idx, p.r_history, p.r_idx, p.r_scale, p.r_scale_inv, s_used);
}

// ---- PTX wrappers (written from the PTX ISA description) -----------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Bounded wait for the phase of parity `parity` to complete.  Returns false if
// the budget ran out (error recorded, abort raised) or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint32_t* err,
                                          uint32_t site, unsigned long long budget_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > budget_ns) {
        record_device_error(err, site);
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// Bulk tensor store of a shared-memory box; clipped to the tensor bounds.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* tm, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_le1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Every bulk store of this thread has finished reading shared memory (its
// global writes may still be in flight: the grid's completion orders them
// before any later kernel's reads).
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA load whose completion is counted on the leader CTA's barrier (bar is a
// shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* tm, int c0, int c1, int c2,
                                                 uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

template <int PAIR>
__device__ __forceinline__ void tmem_alloc_g(uint32_t slot, uint32_t ncols) {
  if constexpr (PAIR == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  } else {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
}

template <int PAIR>
__device__ __forceinline__ void tmem_dealloc_g(uint32_t taddr, uint32_t ncols) {
  if constexpr (PAIR == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
  } else {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
  }
}

// cta_group::2 MMA issued by the leader CTA: A rows 0..127 and B rows 0..BN/2-1
// come from the leader's shared memory, the other halves from the peer's at
// the same offsets; D rows 0..127 land in the leader's TMEM, 128..255 in the peer's.
__device__ __forceinline__ void umma_f8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the barrier at offset `bar` in both CTAs of the pair when all
// prior MMAs of this thread complete.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(uint16_t(3))
      : "memory");
}

__device__ __forceinline__ void umma_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns; lane t of the warp receives row
// (32 * (warp % 4) + t) of the accumulator.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: 8-row x 128-byte atoms stacked along M/N every 1024 bytes
// (stride byte offset), leading byte offset unused for this layout, version 1,
// layout type 2 (128B swizzle).  The tile base is 1024-byte aligned.
__device__ __forceinline__ uint64_t sdesc_k128(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(1) << 16;
  d |= uint64_t(1024 >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// Shared-memory matrix descriptor of an MN-major tile written by TMA with the
// 128-byte swizzle: atoms of 8 K-rows x 128 bytes of M (or N), K-row groups
// every 1024 bytes (stride byte offset), 128-element M/N groups `lbo` bytes
// apart (leading byte offset), version 1, layout type 2.  One 32-deep K step
// of the MMA covers 32 K-rows = 4096 bytes.
__device__ __forceinline__ uint64_t sdesc_mn128(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t(1024 >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// First k-block iteration of stream-K piece s (s may equal sk_ctas: the end).
__device__ __forceinline__ int64_t sk_begin(const MmParams& p, int s) {
  return int64_t(s) * p.sk_iters / p.sk_ctas;
}

// The piece that holds stream-K iteration g: the largest s with sk_begin(s) <= g.
__device__ __forceinline__ int sk_owner(const MmParams& p, int64_t g) {
  return int(((g + 1) * p.sk_ctas + p.sk_iters - 1) / p.sk_iters) - 1;
}

// Unit i of CTA (pair) s in a grid of P: tile t and k-blocks [kb0, kb1).
// A CTA runs its stream-K piece first, then its whole tiles, so that a
// tile's finisher (which holds the tile's first k-blocks at the end of its
// piece) waits for partials that the next pieces wrote at their start, and
// its partial reads overlap the mainloop of its next whole tile.
// False past the CTA's last unit.
__device__ __forceinline__ bool unit_at(const MmParams& p, int s, int P, int i, int& t, int& kb0, int& kb1) {
  int n_sk = 0;
  if (s < p.sk_ctas) {
    const int64_t g0 = sk_begin(p, s), g1 = sk_begin(p, s + 1);
    if (g0 < g1) {
      const int64_t first = g0 / p.k_blocks;
      n_sk = int((g1 - 1) / p.k_blocks - first + 1);
      if (i < n_sk) {
        const int64_t tb = (first + i) * p.k_blocks;
        kb0 = g0 > tb ? int(g0 - tb) : 0;
        kb1 = g1 - tb < p.k_blocks ? int(g1 - tb) : p.k_blocks;
        t = p.dp_tiles + int(first + i);
        return true;
      }
    }
  }
  t = s + (i - n_sk) * P;
  if (t >= p.dp_tiles) return false;
  kb0 = 0;
  kb1 = p.k_blocks;
  return true;
}

__device__ __forceinline__ void decode_tile(const MmParams& p, int t, int& b, int& mt, int& nt) {
  b = t / p.tiles_per_batch;
  const int r = t - b * p.tiles_per_batch;
  const int span = p.group_m * p.n_tiles;
  const int g = r / span;
  const int first_m = g * p.group_m;
  const int gm = min(p.m_tiles - first_m, p.group_m);
  const int rr = r - g * span;
  mt = first_m + rr % gm;
  nt = rr / gm;
}

// One CTA's (pair's) whole life: problem `p` with maps tmA / tmB / tmC, as
// CTA (pair) `cta` of the `ctas` that work on this problem.
template <int BN, int PAIR, int EPI>
__device__ __forceinline__ void mm_body(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmC,
                                        const MmParams& p, const int cta, const int ctas) {
  using C = Cfg<BN, PAIR>;
  constexpr bool kOut8 = (EPI & kEpiOut8) != 0;
  constexpr bool kBias8 = (EPI & kEpiBias8) != 0;
  constexpr int kTileM = kBM * PAIR;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles (the same offset in both CTAs of a pair).
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  // bars[0, S) full, [S, 2S) empty, [2S, 2S+2) tmem_full, [2S+2, 2S+4) tmem_empty, [2S+4] mma_done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 5);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* amax_s = reinterpret_cast<float*>(tmem_slot + 4);  // FP8 output: max |y| per epilogue warp
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * C::kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * C::kStages + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * C::kStages + 4);
  // After the TMEM slot, abort flag and amax slots: never arrived on.
  const uint32_t stall_bar = bar0 + 8u * (2 * C::kStages + 11);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();
  const uint32_t rank = PAIR == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiWarps * PAIR);
    }
    mbar_init(done_bar, 1);
    mbar_init(stall_bar, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(tmA);
    prefetch_tmap(tmB);
    if (p.tma_store) prefetch_tmap(tmC);
  }
  if constexpr (PAIR == 2) cluster_sync();  // the peer's barriers exist before any remote arrive
  if (warp == 1) tmem_alloc_g<PAIR>(smem_u32(tmem_slot), C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_prior_grid();  // inputs, scales and the output buffer belong to earlier work until here
  // FP8 output: lanes 0..17 of warp 1 hold the output ring's history, idx and
  // scale from here to the fold, so the last CTA's fold waits for no loads.
  float ring_v = 0.0f;
  if constexpr (kOut8) {
    if (warp == 1 && lane <= kHistoryLen + 1)
      ring_v = lane < kHistoryLen ? p.r_history[lane] : lane == kHistoryLen ? __int_as_float(*p.r_idx) : *p.r_scale;
  }

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs of a pair) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;  // bit s: stage s armed; its parity
      bool ok = true;
      for (int i = 0; ok; ++i) {
        int t, kb0, kb1;
        if (!unit_at(p, cta, ctas, i, t, kb0, kb1)) break;
        int b, mt, nt;
        decode_tile(p, t, b, mt, nt);
        const int ba = p.a_bcast ? 0 : b;
        const int bb = p.b_bcast ? 0 : b;
        const int arow = mt * kTileM + int(rank) * kBM;
        const int brow = nt * BN + int(rank) * C::kBRows;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort, p.err, kWaitProducerEmpty, p.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + stage * C::kABytes;
          const uint32_t sb = sbase + C::kStages * C::kABytes + stage * C::kBBytes;
          // K-major boxes are [rows][128 K bytes] at (k, row); MN-major boxes
          // are [128 K rows][128 M/N bytes] at (row, k), one per 128 rows.
          uint32_t bar = full_bar(stage);
          if constexpr (PAIR == 1) {
            mbar_arrive_expect_tx(bar, C::kStageBytes);
          } else {
            // Both CTAs' loads complete on the leader's barrier; the leader
            // expects the bytes of both.
            if (leader) mbar_arrive_expect_tx(bar, 2 * C::kStageBytes);
            bar = mapa_shared(bar, 0);
          }
          auto load = [&](uint32_t dst, const CUtensorMap* tm, int c0, int c1, int c2) {
            if constexpr (PAIR == 1) tma_load_3d(dst, tm, c0, c1, c2, bar);
            else tma_load_3d_pair(dst, tm, c0, c1, c2, bar);
          };
          if (p.a_mn) load(sa, tmA, arow, kb * kBK, ba);
          else load(sa, tmA, kb * kBK, arow, ba);
          if (p.b_mn) {
#pragma unroll
            for (int g = 0; g < C::kBRows / 128; ++g) load(sb + g * 16384u, tmB, brow + 128 * g, kb * kBK, bb);
          } else {
            load(sb, tmB, kb * kBK, brow, bb);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // Let every copy armed on this barrier land before shared memory is released.
        for (int s = 0; s < C::kStages; ++s)
          if (armed & (1u << s)) {
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(full_bar(s), (armed_par >> s) & 1u) && globaltimer_ns() - t0 < kWaitBudgetNs) {
            }
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA only) ----------------
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int i = 0;
      bool ok = true;
      const uint32_t sa0 = sbase;
      const uint32_t sb0 = sbase + C::kStages * C::kABytes;
      for (; ok; ++i) {
        int t, kb0, kb1;
        if (!unit_at(p, cta, ctas, i, t, kb0, kb1)) break;
        const int acc = i & 1;
        const uint32_t acc_par = (i >> 1) & 1;
        if (!mbar_wait(tempty_bar(acc), acc_par ^ 1u, abort, p.err, kWaitMmaTmemEmpty, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort, p.err, kWaitMmaFull, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // K-major: +32 bytes along K inside the swizzle atom (+2 in the
          // address field) per MMA.  MN-major: +32 K-rows = 4096 bytes (+256).
          const uint64_t ad = p.a_mn ? sdesc_mn128(sa0 + stage * C::kABytes, 16384u)
                                     : sdesc_k128(sa0 + stage * C::kABytes);
          const uint64_t bd = p.b_mn ? sdesc_mn128(sb0 + stage * C::kBBytes, 16384u)
                                     : sdesc_k128(sb0 + stage * C::kBBytes);
          const uint64_t astep = p.a_mn ? 256u : 2u;
          const uint64_t bstep = p.b_mn ? 256u : 2u;
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            if constexpr (PAIR == 1)
              umma_f8(d, ad + astep * k, bd + bstep * k, p.idesc, (kb != kb0 || k != 0) ? 1u : 0u);
            else
              umma_f8_pair(d, ad + astep * k, bd + bstep * k, p.idesc, (kb != kb0 || k != 0) ? 1u : 0u);
          }
          if constexpr (PAIR == 1) umma_commit(empty_bar(stage));
          else umma_commit_pair(empty_bar(stage));
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (PAIR == 1) umma_commit(tfull_bar(acc));
        else umma_commit_pair(tfull_bar(acc));
      }
      // All MMAs this thread issued are complete before TMEM is released.
      if constexpr (PAIR == 1) umma_commit(done_bar);
      else umma_commit_pair_local(done_bar);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(done_bar, 0) && globaltimer_ns() - t0 < kWaitBudgetNs) {
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9 of each CTA) ----------------
    // Warp w reads TMEM lane quadrant w % 4 (rows 32*(w%4) .. +31 of this
    // CTA's 128-row half) and half (w-2)/4 of the columns.  Two 32-column
    // chunks are loaded per tcgen05.wait::ld; the accumulator is released to
    // the MMA issuer as soon as its last chunk is in registers.  Results leave
    // through 32x32 bf16 TMA stores from two 64B-swizzled staging buffers per
    // warp (rows of 64 bytes, 16-byte unit j of row r at unit j ^ ((r>>1)&3)),
    // or, when output rows are not 16-byte aligned, through guarded stores.
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int half = ew >> 2;
    constexpr int kHalfCols = BN / 2;
    const float sab = __fmul_rn(*p.sinv_a, *p.sinv_b);
    const float bsc = kBias8 ? *p.bias_scale : 0.0f;  // FP8 bias dequantisation factor
    const float s_out = kOut8 ? *p.r_scale : 0.0f;    // FP8 output: the output ring's scale
    float amax = 0.0f;                                 // FP8 output: max |y| of this lane's elements
    const uint32_t stage0 = sbase + C::kStagingOffset + uint32_t(ew) * 2u * kStagingBytes;
    int buf = 0;
    int i = 0;
    constexpr int kChunks = kHalfCols / 32;
    constexpr uint32_t kPieceWarps = uint32_t(kEpiWarps * PAIR);  // arrivals of one piece's partial
    for (;; ++i) {
      int t, kb0, kb1;
      if (!unit_at(p, cta, ctas, i, t, kb0, kb1)) break;
      // A piece that starts inside the tile hands its partial on; the piece
      // with k-block 0 of a tile it does not finish adds the later pieces'
      // partials, pieces cta+1 .. last_piece.
      const bool writer = kb0 > 0;
      const bool finisher = kb0 == 0 && kb1 < p.k_blocks;
      const int last_piece =
          finisher ? sk_owner(p, int64_t(t - p.dp_tiles) * p.k_blocks + p.k_blocks - 1) : cta;
      const int acc = i & 1;
      const uint32_t acc_par = (i >> 1) & 1;
      // (Testing: with the stall site set here, the wait is on a barrier that
      // nothing completes, so it runs out and the abort path runs.)
      const bool stall = p.stall == kWaitEpilogueTmemFull;
      if (!mbar_wait(stall ? stall_bar : tfull_bar(acc), stall ? 0u : acc_par, abort, p.err, kWaitEpilogueTmemFull,
                     p.wait_ns))
        break;
      tc_fence_after();
      int b, mt, nt;
      decode_tile(p, t, b, mt, nt);
      // Chunk cc of this warp's part of piece q's float32 partial: 32 rows x
      // 32 columns as [j][lane] float4, so each store or load instruction of
      // the warp covers 512 contiguous bytes.
      auto slot = [&](int q, int cc) {
        return reinterpret_cast<float4*>(p.ws + (size_t(q) * PAIR + rank) * size_t(kBM * BN) +
                                         size_t(ew * kChunks + cc) * 1024) + lane;
      };
      if (finisher && lane == 0) {
        // Wait (bounded) until every warp of every later piece of this tile has published its partial.
        const unsigned long long w0 = globaltimer_ns();
        for (int q = cta + 1; q <= last_piece; ++q) {
          uint32_t seen = 0;
          while (true) {
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(p.flags + q) : "memory");
            if (seen >= kPieceWarps) break;
            if (*abort || globaltimer_ns() - w0 > p.wait_ns) {
              record_device_error(p.err, kWaitSplitK);
              *abort = 1;
              break;
            }
          }
        }
      }
      if (finisher) {
        __syncwarp();
        __threadfence();
      }
      const int m0 = mt * kTileM + int(rank) * kBM + quad * 32;
      const uint32_t tbase = tmem_base + (uint32_t(quad * 32) << 16) + uint32_t(acc * BN + half * kHalfCols);
      const int nbase = nt * BN + half * kHalfCols;
      // This warp's bias, four columns per lane (lane l: nbase + 4l .. 4l+3),
      // read once per tile; emit() takes a chunk's 32 values from 8 lanes by
      // shuffle.  (Broadcast loads of the same values in every chunk cost a
      // K=1536 GEMM about 28% of its time.)
      const bool has_bias = kBias8 || p.bias != nullptr;
      float4 bias_l = make_float4(0.f, 0.f, 0.f, 0.f);
      if (has_bias && lane < kHalfCols / 4) {
        const int c4 = nbase + 4 * lane;
        if constexpr (kBias8) {
          bias_l = bias8_4(p, c4, bsc);
        } else if (p.bias_vec && c4 + 3 < p.N) {
          bias_l = __ldg(reinterpret_cast<const float4*>(p.bias + c4));
        } else {
          bias_l.x = c4 < p.N ? __ldg(p.bias + c4) : 0.f;
          bias_l.y = c4 + 1 < p.N ? __ldg(p.bias + c4 + 1) : 0.f;
          bias_l.z = c4 + 2 < p.N ? __ldg(p.bias + c4 + 2) : 0.f;
          bias_l.w = c4 + 3 < p.N ? __ldg(p.bias + c4 + 3) : 0.f;
        }
      }
      const uint32_t release_bar = PAIR == 1 ? tempty_bar(acc) : mapa_shared(tempty_bar(acc), 0);
      bool released = false;
      auto release = [&]() {
        // Last TMEM read of this tile for this warp: hand the accumulator back.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(release_bar);
        released = true;
      };
      // One 32 x 32 chunk at output columns n0 (this lane's row): scale, bias,
      // one bf16 rounding, store.
      auto emit = [&](int n0, const uint32_t(&v)[32]) {
        if (m0 >= p.M) return;  // warp-uniform: rows beyond M (pair peer of a short last tile)
        const bool full = n0 + 32 <= p.N;
        const bool row_ok = m0 + lane < p.M;
        uint32_t packed[16];  // bf16 pairs, or (FP8 output) code quads in [0, 8)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
          if (has_bias) {  // warp-uniform
            const int src = ((n0 - nbase) >> 5) * 8 + j;
            bv.x = __shfl_sync(0xFFFFFFFFu, bias_l.x, src);
            bv.y = __shfl_sync(0xFFFFFFFFu, bias_l.y, src);
            bv.z = __shfl_sync(0xFFFFFFFFu, bias_l.z, src);
            bv.w = __shfl_sync(0xFFFFFFFFu, bias_l.w, src);
          }
          float y0 = __uint_as_float(v[4 * j + 0]), y1 = __uint_as_float(v[4 * j + 1]);
          float y2 = __uint_as_float(v[4 * j + 2]), y3 = __uint_as_float(v[4 * j + 3]);
          fma2(y0, y1, sab, bv.x, bv.y);  // acc * sinv_a*sinv_b + bias, one rounding each
          fma2(y2, y3, sab, bv.z, bv.w);
          if constexpr (kOut8) {
            // amax over this lane's in-range elements (NaN ignored), then the
            // codes of y * s_out.
            if (row_ok && full) {  // full: warp-uniform, so no per-column checks
              amax = fmaxf(amax, fmaxf(fmaxf(fabsf(y0), fabsf(y1)), fmaxf(fabsf(y2), fabsf(y3))));
            } else if (row_ok) {
              const int nn = n0 + 4 * j;
              amax = fmaxf(amax, nn < p.N ? fabsf(y0) : 0.f);
              amax = fmaxf(amax, nn + 1 < p.N ? fabsf(y1) : 0.f);
              amax = fmaxf(amax, nn + 2 < p.N ? fabsf(y2) : 0.f);
              amax = fmaxf(amax, nn + 3 < p.N ? fabsf(y3) : 0.f);
            }
            packed[j] = p.out_fmt == FP8_E5M2 ? cvt4<FP8_E5M2>(y0, y1, y2, y3, s_out)
                                              : cvt4<FP8_E4M3>(y0, y1, y2, y3, s_out);
          } else {
            const __nv_bfloat162 h01 = __floats2bfloat162_rn(y0, y1);
            const __nv_bfloat162 h23 = __floats2bfloat162_rn(y2, y3);
            packed[2 * j] = *reinterpret_cast<const uint32_t*>(&h01);
            packed[2 * j + 1] = *reinterpret_cast<const uint32_t*>(&h23);
          }
        }
        if constexpr (kOut8) {
          if (p.tma_store) {
            // 32 x 32 codes through a TMA store (clipped to M and N) from the
            // first 1 KB of a staging buffer, 32B swizzle: 16-byte unit u of
            // row r at unit u ^ ((r >> 2) & 1), conflict-free for the warp.
            const uint32_t sbuf = stage0 + uint32_t(buf) * kStagingBytes;
            if (lane == 0) bulk_wait_read_le1();
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const uint32_t addr = sbuf + uint32_t(lane) * 32u + uint32_t((u ^ ((lane >> 2) & 1)) * 16);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(packed[4 * u]),
                           "r"(packed[4 * u + 1]), "r"(packed[4 * u + 2]), "r"(packed[4 * u + 3])
                           : "memory");
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(tmC, sbuf, n0, m0, b);
              bulk_commit();
            }
            buf ^= 1;
            return;
          }
          // Rows not 16-byte aligned: the chunk is staged in the same
          // layout, then written row by row, lane l taking column n0 + l, so
          // each store instruction covers 32 contiguous bytes of one row.
          const uint32_t sbuf = stage0 + uint32_t(buf) * kStagingBytes;
          __syncwarp();  // every lane has read this buffer's previous chunk
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint32_t addr = sbuf + uint32_t(lane) * 32u + uint32_t((u ^ ((lane >> 2) & 1)) * 16);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(packed[4 * u]),
                         "r"(packed[4 * u + 1]), "r"(packed[4 * u + 2]), "r"(packed[4 * u + 3])
                         : "memory");
          }
          __syncwarp();
          const bool col_ok = n0 + lane < p.N;
          uint8_t* obase = p.out8 + int64_t(b) * p.c_stride + int64_t(m0) * p.N + n0 + lane;
#pragma unroll 4
          for (int rr = 0; rr < 32; ++rr) {
            const uint32_t addr =
                sbuf + uint32_t(rr) * 32u + uint32_t((((lane >> 4) ^ ((rr >> 2) & 1)) << 4) + (lane & 15));
            uint16_t v16;
            asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v16) : "r"(addr) : "memory");
            if (col_ok && m0 + rr < p.M) obase[int64_t(rr) * p.N] = uint8_t(v16);
          }
          buf ^= 1;
          return;
        }
        const uint32_t sbuf = stage0 + uint32_t(buf) * kStagingBytes;
        // The buffer's previous TMA store has read it (checked after the math,
        // so the wait overlaps it).
        if (p.tma_store && lane == 0) bulk_wait_read_le1();
        __syncwarp();
        // 16-byte unit u of this lane's 64-byte row holds columns 8u .. 8u+7,
        // at unit position u ^ ((lane >> 1) & 3).
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t addr = sbuf + uint32_t(lane) * 64u + uint32_t((u ^ ((lane >> 1) & 3)) * 16);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(packed[4 * u]),
                       "r"(packed[4 * u + 1]), "r"(packed[4 * u + 2]), "r"(packed[4 * u + 3])
                       : "memory");
        }
        if (p.tma_store) {
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(tmC, sbuf, n0, m0, b);
            bulk_commit();
          }
        } else {
          // Rows not 16-byte aligned: the chunk staged in the same swizzled
          // layout is written row by row, lane l taking column n0 + l, so
          // each store instruction covers 64 contiguous bytes.
          __syncwarp();
          const bool col_ok = n0 + lane < p.N;
          uint16_t* obase = p.out + int64_t(b) * p.c_stride + int64_t(m0) * p.N + n0 + lane;
#pragma unroll 4
          for (int rr = 0; rr < 32; ++rr) {
            const uint32_t addr = sbuf + uint32_t(rr) * 64u + uint32_t((((lane >> 3) ^ ((rr >> 1) & 3)) << 4)) +
                                  uint32_t((lane & 7) << 1);
            uint16_t v16;
            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v16) : "r"(addr) : "memory");
            if (col_ok && m0 + rr < p.M) obase[int64_t(rr) * p.N] = v16;
          }
        }
        buf ^= 1;
      };
      auto add4 = [](uint32_t* v, const float4& w) {
        v[0] = __float_as_uint(__uint_as_float(v[0]) + w.x);
        v[1] = __float_as_uint(__uint_as_float(v[1]) + w.y);
        v[2] = __float_as_uint(__uint_as_float(v[2]) + w.z);
        v[3] = __float_as_uint(__uint_as_float(v[3]) + w.w);
      };
#pragma unroll 1
      for (int c = 0; c < kChunks; c += 2) {
        if (nbase + c * 32 >= p.N) break;  // warp-uniform: the rest of this half is beyond N
        const bool two = c + 1 < kChunks && nbase + (c + 1) * 32 < p.N;
        const bool last_pair = c + 2 >= kChunks || nbase + (c + 2) * 32 >= p.N;
        if (finisher) {
          // Per chunk: the next piece's partial is requested (8 independent
          // 512-byte warp loads) before the TMEM read; any further pieces are
          // added after it, in piece order.
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h == 1 && !two) break;
            float4 pv[8];
            const float4* src = slot(cta + 1, c + h);
#pragma unroll
            for (int j = 0; j < 8; ++j) pv[j] = __ldcg(src + 32 * j);
            uint32_t r[32];
            tmem_ld32_nowait(tbase + uint32_t((c + h) * 32), r);
            tmem_wait_ld();
            if (last_pair && (h == 1 || !two)) release();
#pragma unroll
            for (int j = 0; j < 8; ++j) add4(r + 4 * j, pv[j]);
            for (int q = cta + 2; q <= last_piece; ++q) {
              const float4* src2 = slot(q, c + h);
#pragma unroll
              for (int j = 0; j < 8; ++j) add4(r + 4 * j, __ldcg(src2 + 32 * j));
            }
            emit(nbase + (c + h) * 32, r);
          }
          continue;
        }
        uint32_t r[2][32];
        tmem_ld32_nowait(tbase + uint32_t(c * 32), r[0]);
        if (two) tmem_ld32_nowait(tbase + uint32_t((c + 1) * 32), r[1]);
        tmem_wait_ld();
        if (last_pair) release();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && !two) break;
          if (writer) {
            float4* dst = slot(cta, c + h);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              __stcg(dst + 32 * j, make_float4(__uint_as_float(r[h][4 * j]), __uint_as_float(r[h][4 * j + 1]),
                                               __uint_as_float(r[h][4 * j + 2]), __uint_as_float(r[h][4 * j + 3])));
          } else {
            emit(nbase + (c + h) * 32, r[h]);
          }
        }
      }
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(release_bar);
      }
      if (writer) {
        __threadfence();  // this warp's partial stores are visible before its arrival
        __syncwarp();
        if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.flags + cta) : "memory");
      } else if (finisher) {
        __syncwarp();
        if (lane == 0) {
          // Each finishing warp counts itself on every piece it read; the last
          // of a piece's writer and reader warps clears its flag for the next call.
          for (int q = cta + 1; q <= last_piece; ++q) {
            const uint32_t old = atomicAdd(p.flags + q, 1u);
            if (old == 2u * kPieceWarps - 1u) atomicExch(p.flags + q, 0u);
          }
        }
      }
    }
    if constexpr (kOut8) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) amax_s[ew] = amax;
    }
    // The staging buffers are released once the stores have read them; waiting
    // for the global writes too kept every CTA alive ~0.4 us longer.
    if (p.tma_store && lane == 0) bulk_wait_read_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kOut8) {
    if (warp == 1) {
      // The staging buffers are free: every epilogue warp waited for its
      // stores before the barrier above.
      float* ring_s = reinterpret_cast<float*>(smem + C::kStagingOffset);
      if (lane <= kHistoryLen + 1) ring_s[lane] = ring_v;
      __syncwarp();
      if (lane == 0) out8_ticket_fold(p, amax_s, ring_s);
      __syncwarp();
    }
  }
  // A pair leaves together: the leader's MMAs read the peer's shared memory
  // and write the peer's TMEM until done_bar fired.
  if constexpr (PAIR == 2) cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_g<PAIR>(tmem_base, C::kTmemCols);
}

template <int BN, int PAIR, int EPI>
__global__ void __launch_bounds__(kThreadsMM, 1)
    mm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ MmParams p) {
  mm_body<BN, PAIR, EPI>(&tmA, &tmB, &tmC, p, int(blockIdx.x) / PAIR, int(gridDim.x) / PAIR);
}

// Two independent GEMMs in one persistent launch (the dX and dW GEMMs of a
// linear's backward): CTAs (pairs) [0, split) work on problem 0 and the rest
// on problem 1, each set over its own tiles, so a problem with too few tiles
// to fill the GPU shares it with the other instead of leaving SMs idle.
template <int BN, int PAIR>
__global__ void __launch_bounds__(kThreadsMM, 1)
    mm_fp8_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ MmParams p0,
                       const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                       const __grid_constant__ CUtensorMap tmC1, const __grid_constant__ MmParams p1, const int split) {
  const int g = int(blockIdx.x) / PAIR;
  if (g < split) mm_body<BN, PAIR, 0>(&tmA0, &tmB0, &tmC0, p0, g, split);
  else mm_body<BN, PAIR, 0>(&tmA1, &tmB1, &tmC1, p1, g - split, int(gridDim.x) / PAIR - split);
}

// K == 0: Y = bf16(bias) or 0.
// Bias value of column n: float32, dequantised FP8, or 0 without a bias.
__device__ __forceinline__ float bias_at(const MmParams& p, int64_t n) {
  if (p.bias8 != nullptr) return __fmul_rn(fp8_value(p.bias8[n], p.bias_fmt), *p.bias_scale);
  return p.bias != nullptr ? p.bias[n] : 0.0f;
}

__global__ void mm_bias_only_kernel(const MmParams p, int64_t M, int64_t N, int64_t batch) {
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  const int64_t total = batch * M * N;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t b = i / (M * N), r = i - b * M * N, n = r % N;
    const __nv_bfloat16 h = __float2bfloat16_rn(bias_at(p, n));
    p.out[b * p.c_stride + r] = *reinterpret_cast<const uint16_t*>(&h);
  }
}

// FP8 output with K == 0 (y = bias) or an empty output (amax 0): one CTA
// writes the codes, reduces max |y| and commits the output ring, so every
// call still adds exactly one history entry.
__global__ void __launch_bounds__(256) mm_out8_small_kernel(const MmParams p, int64_t M, int64_t N, int64_t batch) {
  __shared__ float warp_max[8];
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  const float s = *p.r_scale;
  const int64_t total = batch * M * N;
  float amax = 0.0f;
  for (int64_t i = threadIdx.x; i < total; i += blockDim.x) {
    const int64_t b = i / (M * N), r = i - b * M * N, n = r % N;
    const float y = bias_at(p, n);
    amax = fmaxf(amax, fabsf(y));
    p.out8[b * p.c_stride + r] = p.out_fmt == FP8_E5M2 ? cvt_one<FP8_E5M2>(y, s) : cvt_one<FP8_E4M3>(y, s);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x != 0) return;
  float a = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) a = fmaxf(a, warp_max[w]);
  if (p.amax_out != nullptr) {
    *p.amax_out = a;
    *p.r_scale_inv = __frcp_rn(s);
    return;
  }
  float hist[kHistoryLen];
#pragma unroll
  for (int i = 0; i < kHistoryLen; ++i) hist[i] = p.r_history[i];
  if (p.out_fmt == FP8_E5M2)
    ring_commit<FP8_E5M2>(a, hist, *p.r_idx, p.r_history, p.r_idx, p.r_scale, p.r_scale_inv, s);
  else
    ring_commit<FP8_E4M3>(a, hist, *p.r_idx, p.r_history, p.r_idx, p.r_scale, p.r_scale_inv, s);
}

// ---- host side -----------------------------------------------------------------

// 3-D map over uint8 [batch, rows, K] with a box of [1, box_rows, 128], 128B swizzle.
bool make_map(CUtensorMap* m, const uint8_t* base, int64_t K, int64_t rows, int64_t batch, int64_t bstride,
              int box_rows) {
  const uint64_t dims[3] = {uint64_t(K), uint64_t(rows), uint64_t(batch)};
  const uint64_t strides[2] = {uint64_t(K), uint64_t(batch > 1 ? bstride : K * rows)};
  const uint32_t box[3] = {uint32_t(kBK), uint32_t(box_rows), 1u};
  return encode_tiled_cached(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// 3-D map over an MN-major uint8 operand [batch, K, mn] (mn contiguous) with a
// box of [1, 128 K rows, 128 mn bytes], 128B swizzle.
bool make_map_mn(CUtensorMap* m, const uint8_t* base, int64_t K, int64_t mn, int64_t batch, int64_t bstride) {
  const uint64_t dims[3] = {uint64_t(mn), uint64_t(K), uint64_t(batch)};
  const uint64_t strides[2] = {uint64_t(mn), uint64_t(batch > 1 ? bstride : K * mn)};
  const uint32_t box[3] = {128u, uint32_t(kBK), 1u};
  return encode_tiled_cached(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// 3-D map over the bf16 output [batch, M, N] with a 32x32 box, 64B swizzle
// (the staging-buffer layout the epilogue writes).
bool make_out_map(CUtensorMap* m, uint16_t* base, int64_t M, int64_t N, int64_t batch, int64_t c_stride);

// 3-D map over FP8 output codes [batch, M, N] with a 32x32 box, 32B swizzle.
bool make_out8_map(CUtensorMap* m, uint8_t* base, int64_t M, int64_t N, int64_t batch, int64_t c_stride) {
  const uint64_t dims[3] = {uint64_t(N), uint64_t(M), uint64_t(batch)};
  const uint64_t strides[2] = {uint64_t(N), uint64_t(batch > 1 ? c_stride : M * N)};
  const uint32_t box[3] = {32u, 32u, 1u};
  return encode_tiled_cached(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

bool make_out_map(CUtensorMap* m, uint16_t* base, int64_t M, int64_t N, int64_t batch, int64_t c_stride) {
  const uint64_t dims[3] = {uint64_t(N), uint64_t(M), uint64_t(batch)};
  const uint64_t strides[2] = {uint64_t(N * 2), uint64_t((batch > 1 ? c_stride : M * N) * 2)};
  const uint32_t box[3] = {32u, 32u, 1u};
  return encode_tiled_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box,
                             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int BN, int PAIR, int EPI = 0>
bool ensure_smem_attr() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(mm_fp8_kernel<BN, PAIR, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<BN, PAIR>::kSmemBytes) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

// CTA pairs that can be resident at once (one pair per two SMs at best).
template <int BN>
int max_pairs(int sms) {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return sms / 2;
  if (cached[dev] == 0) {
    if (!ensure_smem_attr<BN, 2>()) return sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2));
    cfg.blockDim = dim3(kThreadsMM);
    cfg.dynamicSmemBytes = Cfg<BN, 2>::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, mm_fp8_kernel<BN, 2, 0>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = sms / 2;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

// Launch shape: tile width, CTA pairing, grid size in CTAs (pairs), whole
// tiles, stream-K pieces and the workspace the pieces need.
struct MmChoice {
  int bn, pair, grid, dp_tiles, sk_ctas;
  size_t ws_bytes;
  double cost;  // modelled time, microseconds
};

constexpr int kMaxPieces = 256;             // flag words in the workspace's first 1024 bytes
constexpr size_t kFlagBytes = 4 * kMaxPieces;

// Workspace of a stream-K launch: 1024 bytes of per-piece arrival counters,
// then one float32 128 x BN partial per piece and CTA of a pair.
size_t sk_ws_bytes(int pieces, int bn, int pair) {
  return pieces > 0 ? kFlagBytes + size_t(pieces) * size_t(pair) * kBM * size_t(bn) * 4 : 0;
}

// One validated GEMM: its arguments and the parameters that do not depend on
// the launch shape.
struct MmProblem {
  const uint8_t* A;
  const uint8_t* B;
  int64_t M, N, K, batch;
  const int64_t* strides;
  bool nothing;  // M == 0 or N == 0: no output
  int epi;       // kEpiOut8 | kEpiBias8 bits: which epilogue variant runs
  MmParams p;
};

// Tensor maps and tile parameters of problem q for the launch shape c.
template <int BN, int PAIR>
int prepare_mm(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
               const int64_t* strides, MmParams& p, const MmChoice& c, void* ws, CUtensorMap& ta, CUtensorMap& tb,
               CUtensorMap& tc) {
  const int64_t ba = (batch > 1 && strides[0] != 0) ? batch : 1;
  const int64_t bb = (batch > 1 && strides[1] != 0) ? batch : 1;
  const bool okA = p.a_mn ? make_map_mn(&ta, A, K, M, ba, ba > 1 ? strides[0] : 0)
                          : make_map(&ta, A, K, M, ba, ba > 1 ? strides[0] : 0, kBM);
  const bool okB = p.b_mn ? make_map_mn(&tb, B, K, N, bb, bb > 1 ? strides[1] : 0)
                          : make_map(&tb, B, K, N, bb, bb > 1 ? strides[1] : 0, BN / PAIR);
  if (!okA || !okB) return FP8_ERR_CUDA;
  memset(&tc, 0, sizeof(tc));
  if (p.tma_store && !(p.out8 != nullptr ? make_out8_map(&tc, p.out8, M, N, batch, p.c_stride)
                                         : make_out_map(&tc, p.out, M, N, batch, p.c_stride)))
    return FP8_ERR_CUDA;
  p.a_bcast = ba == 1;
  p.b_bcast = bb == 1;
  p.m_tiles = int((M + kBM * PAIR - 1) / (kBM * PAIR));
  p.n_tiles = int((N + BN - 1) / BN);
  p.tiles_per_batch = p.m_tiles * p.n_tiles;
  p.tiles_total = int(p.tiles_per_batch * batch);
  p.dp_tiles = c.dp_tiles;
  p.sk_ctas = c.sk_ctas;
  p.sk_iters = int64_t(p.tiles_total - c.dp_tiles) * p.k_blocks;
  if (c.sk_ctas > 0) {
    p.flags = static_cast<uint32_t*>(ws);
    p.ws = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kFlagBytes);
  }
  p.group_m = 8;
  p.idesc |= (uint32_t(BN >> 3) << 17) | (uint32_t((kBM * PAIR) >> 4) << 24);
  return FP8_OK;
}

template <int BN, int PAIR, int EPI>
int launch_mm_epi(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
                  const int64_t* strides, MmParams p, const MmChoice& c, void* ws, cudaStream_t st) {
  CUtensorMap ta, tb, tc;
  const int rc = prepare_mm<BN, PAIR>(A, B, M, N, K, batch, strides, p, c, ws, ta, tb, tc);
  if (rc != FP8_OK) return rc;
  if (!ensure_smem_attr<BN, PAIR, EPI>()) return FP8_ERR_CUDA;
  const cudaError_t e = launch_pdl(mm_fp8_kernel<BN, PAIR, EPI>, dim3(PAIR * std::max(1, c.grid)), dim3(kThreadsMM),
                                   Cfg<BN, PAIR>::kSmemBytes, st, PAIR, ta, tb, tc, p);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

template <int BN, int PAIR>
int launch_mm(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
              const int64_t* strides, const MmParams& p, int epi, const MmChoice& c, void* ws, cudaStream_t st) {
  switch (epi) {
    case 0: return launch_mm_epi<BN, PAIR, 0>(A, B, M, N, K, batch, strides, p, c, ws, st);
    case kEpiOut8: return launch_mm_epi<BN, PAIR, kEpiOut8>(A, B, M, N, K, batch, strides, p, c, ws, st);
    case kEpiBias8: return launch_mm_epi<BN, PAIR, kEpiBias8>(A, B, M, N, K, batch, strides, p, c, ws, st);
    default: return launch_mm_epi<BN, PAIR, kEpiOut8 | kEpiBias8>(A, B, M, N, K, batch, strides, p, c, ws, st);
  }
}

template <int BN, int PAIR>
bool ensure_pair_smem_attr() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(mm_fp8_pair_kernel<BN, PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<BN, PAIR>::kSmemBytes) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

// Two problems in one launch: c0.grid CTAs (pairs) on problem 0, c1.grid on
// problem 1, whole tiles only.
template <int BN, int PAIR>
int launch_pair(MmProblem& q0, const MmChoice& c0, MmProblem& q1, const MmChoice& c1, cudaStream_t st) {
  CUtensorMap ta0, tb0, tc0, ta1, tb1, tc1;
  MmParams p0 = q0.p, p1 = q1.p;
  int rc = prepare_mm<BN, PAIR>(q0.A, q0.B, q0.M, q0.N, q0.K, q0.batch, q0.strides, p0, c0, nullptr, ta0, tb0, tc0);
  if (rc != FP8_OK) return rc;
  rc = prepare_mm<BN, PAIR>(q1.A, q1.B, q1.M, q1.N, q1.K, q1.batch, q1.strides, p1, c1, nullptr, ta1, tb1, tc1);
  if (rc != FP8_OK) return rc;
  if (!ensure_pair_smem_attr<BN, PAIR>()) return FP8_ERR_CUDA;
  const cudaError_t e =
      launch_pdl(mm_fp8_pair_kernel<BN, PAIR>, dim3(PAIR * (c0.grid + c1.grid)), dim3(kThreadsMM),
                 Cfg<BN, PAIR>::kSmemBytes, st, PAIR, ta0, tb0, tc0, p0, ta1, tb1, tc1, p1, c0.grid);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// Launch-shape choice by a time model in microseconds, over 256-wide tiles
// on CTA pairs or single CTAs, single CTAs with 128- and 64-wide tiles and,
// given a workspace, a stream-K tail.  (128-wide tiles on CTA pairs run the
// same waves as on single CTAs and were never faster.)  Fitted to graph-timed B200 runs of every shape at square
// sizes 512-2048 and the 1.2B-model linears (M 512-8192):
//   * whole tiles run in waves of `slots`; one k-block of one wave takes
//     `s` (0.35 us for 128 x 64 tiles up to 0.41-0.44 us for 256-wide ones:
//     the mainloop is bound by operand traffic into the SM, so wider tiles
//     do more work per byte), and a launch costs a fixed `I` (set-up, first
//     loads, the last tile's epilogue: more columns, more epilogue);
//   * stream-K (data-parallel + two-tile stream-K): all but the last full
//     wave stay whole tiles; the k-blocks of the rest are dealt evenly to the
//     pieces.  A piece costs its k-blocks plus the fix-up measured on B200
//     for a 128 x 256 float32 partial: about 4 us to write it, fence and
//     flag it, and about 5 us per extra piece for the finisher's wait and
//     read (half that for 128-wide and narrower tiles: the waits and fences
//     do not shrink with a 64-wide partial).  So stream-K pays off only
//     where a part of a wave idles for well over 10 us: small outputs with
//     long K.
MmChoice choose_mm(int64_t M, int64_t N, int64_t K, int64_t batch, int sms, bool b_mn, size_t ws_limit) {
  struct Opt {
    int bn, pair;
    double s, fixed;  // us per k-block of a wave; us per launch
  };
  const Opt opts[4] = {{256, 2, 0.41, 5.1}, {256, 1, 0.44, 4.6}, {128, 1, 0.37, 3.5}, {64, 1, 0.35, 3.3}};
  constexpr int kMinIters = 4;  // k-blocks per piece, at least
  const int64_t kb = (K + kBK - 1) / kBK;
  MmChoice best{256, 1, 1, 0, 0, 0, 0.0};
  double best_cost = 1e300;
  for (const Opt& o : opts) {
    if (o.pair == 2 && M <= kBM) continue;  // the second CTA would hold no rows
    if (b_mn && o.bn / o.pair < 128) continue;
    const int slots = o.pair == 2 ? max_pairs<256>(sms) : sms;
    const int64_t tiles = ((M + kBM * o.pair - 1) / (kBM * o.pair)) * ((N + o.bn - 1) / o.bn) * batch;
    const double t_write = 4.0 * (std::max(o.bn, 128) / 256.0), t_read = 5.0 * (std::max(o.bn, 128) / 256.0);
    const double dp_cost = o.fixed + double((tiles + slots - 1) / slots) * double(kb) * o.s;
    if (dp_cost < best_cost) {
      best_cost = dp_cost;
      best = MmChoice{o.bn, o.pair, int(std::min<int64_t>(tiles, slots)), int(tiles), 0, 0, dp_cost};
    }
    if (ws_limit == 0 || tiles % slots == 0 || slots > kMaxPieces || kb < 2 * kMinIters) continue;
    const int64_t full = tiles / slots;
    const int64_t dp = full >= 1 ? (full - 1) * slots : 0;
    const int64_t T = tiles - dp;
    const int64_t W = T * kb;
    int64_t cands[6] = {slots, 2 * T, 3 * T, 4 * T, 5 * T, 6 * T};
    for (int64_t pieces : cands) {
      pieces = std::min<int64_t>(pieces, slots);
      pieces = std::min<int64_t>(pieces, W / kMinIters);
      if (pieces < 2) continue;
      const int64_t L = W / pieces;
      if (W % pieces == 0 && L % kb == 0) continue;  // every piece whole tiles: the data-parallel case
      const int64_t iters = (W + pieces - 1) / pieces;
      const int64_t span = std::min<int64_t>(pieces, (kb - 1 + L - 1) / L + 1);  // pieces a tile can touch
      const double cost = o.fixed + double(dp / slots) * double(kb) * o.s + double(iters) * o.s + t_write +
                          double(span - 1) * t_read;
      const size_t wsb = sk_ws_bytes(int(pieces), o.bn, o.pair);
      if (wsb > ws_limit) continue;
      if (cost < best_cost) {
        best_cost = cost;
        best = MmChoice{o.bn, o.pair, int(dp > 0 ? slots : pieces), int(dp), int(pieces), wsb, cost};
      }
    }
  }
  return best;
}

}  // namespace
}  // namespace fp8ds

using namespace fp8ds;

namespace fp8ds {
namespace {

// fp8_mm_ex's epilogue options beyond fp8_mm's: FP8 bias codes and FP8 output.
struct MmEpilogue {
  const uint8_t* bias8;     // FP8 bias codes [N] (bias_scale set), else null
  const float* bias_scale;  // their dequantisation factor (device scalar)
  int out_kind;             // fp8_mm_out
  uint8_t* out8;            // FP8 output codes (out_kind != FP8_MM_OUT_BF16)
  fp8_ring ring;            // the FP8 output's ring
  float* amax_out;          // data-parallel shard: amax out, no fold
};

int mm_validate(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
                const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b, const float* bias,
                uint16_t* out_bf16, MmProblem& q, const MmEpilogue* ex = nullptr) {
  if (M < 0 || N < 0 || K < 0 || batch < 1) return FP8_ERR_INVALID_ARG;
  const bool bias8 = ex != nullptr && ex->bias8 != nullptr;
  const bool out8 = ex != nullptr && ex->out_kind != FP8_MM_OUT_BF16;
  const int known = FP8_MM_A_E5M2 | FP8_MM_B_E5M2 | FP8_MM_A_MN_MAJOR | FP8_MM_B_MN_MAJOR |
                    (bias8 ? FP8_MM_BIAS_E5M2 : 0);
  if ((layout & ~known) != FP8_MM_NT) return FP8_ERR_INVALID_ARG;
  if (ex != nullptr && ex->out_kind != FP8_MM_OUT_BF16 && ex->out_kind != FP8_MM_OUT_E4M3 &&
      ex->out_kind != FP8_MM_OUT_E5M2)
    return FP8_ERR_INVALID_ARG;
  if (bias8 && (ex->bias_scale == nullptr || bias != nullptr)) return FP8_ERR_INVALID_ARG;
  if (out8) {
    const fp8_ring& r = ex->ring;
    if ((ex->out8 == nullptr && M > 0 && N > 0) || out_bf16 != nullptr) return FP8_ERR_INVALID_ARG;
    if (!r.history || !r.idx || !r.scale || !r.scale_inv || !r.scratch) return FP8_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(r.scratch) % 8 != 0) return FP8_ERR_UNSUPPORTED;
  }
  if (ex != nullptr && ex->amax_out != nullptr && !out8) return FP8_ERR_INVALID_ARG;
  const bool a_mn = (layout & FP8_MM_A_MN_MAJOR) != 0;
  const bool b_mn = (layout & FP8_MM_B_MN_MAJOR) != 0;
  if (batch > 1 && strides == nullptr) return FP8_ERR_INVALID_ARG;
  if (batch > 1 && (strides[0] < 0 || strides[1] < 0 || strides[2] < 0)) return FP8_ERR_INVALID_ARG;
  q = MmProblem{};
  q.A = A;
  q.B = B;
  q.M = M;
  q.N = N;
  q.K = K;
  q.batch = batch;
  q.strides = strides;
  q.nothing = M == 0 || N == 0;
  q.epi = (out8 ? kEpiOut8 : 0) | (bias8 ? kEpiBias8 : 0);
  MmParams& p = q.p;
  const WaitCfg wc = wait_cfg();
  p.wait_ns = wc.budget_ns;
  p.stall = wc.stall_site;
  const int64_t c_stride = batch > 1 ? strides[2] : M * N;
  p.c_stride = c_stride;
  if (out8) {
    p.out_fmt = ex->out_kind == FP8_MM_OUT_E5M2 ? FP8_E5M2 : FP8_E4M3;
    p.out8 = ex->out8;
    p.r_history = ex->ring.history;
    p.r_idx = ex->ring.idx;
    p.r_scale = ex->ring.scale;
    p.r_scale_inv = ex->ring.scale_inv;
    p.r_scratch = ex->ring.scratch;
    p.amax_out = ex->amax_out;
  }
  if (bias8) {
    p.bias8 = ex->bias8;
    p.bias_scale = ex->bias_scale;
    p.bias_fmt = (layout & FP8_MM_BIAS_E5M2) ? FP8_E5M2 : FP8_E4M3;
  }
  if (q.nothing) return FP8_OK;  // nothing to compute (an FP8 output still folds amax 0)
  if ((!out8 && out_bf16 == nullptr) || sinv_a == nullptr || sinv_b == nullptr) return FP8_ERR_INVALID_ARG;
  if (K > 0 && (A == nullptr || B == nullptr)) return FP8_ERR_INVALID_ARG;
  if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2 || batch > 65535) return FP8_ERR_UNSUPPORTED;
  if (K % 16 != 0) return FP8_ERR_UNSUPPORTED;
  if ((a_mn && M % 16 != 0) || (b_mn && N % 16 != 0)) return FP8_ERR_UNSUPPORTED;  // MN-major row pitch
  if (!out8 && reinterpret_cast<uintptr_t>(out_bf16) % 2 != 0) return FP8_ERR_UNSUPPORTED;
  if (K > 0) {
    if (reinterpret_cast<uintptr_t>(A) % 16 != 0 || reinterpret_cast<uintptr_t>(B) % 16 != 0)
      return FP8_ERR_UNSUPPORTED;
    if (batch > 1 && ((strides[0] % 16) != 0 || (strides[1] % 16) != 0)) return FP8_ERR_UNSUPPORTED;
  }
  p.M = int(M);
  p.N = int(N);
  p.K = int(K);
  p.k_blocks = int((K + kBK - 1) / kBK);
  p.sinv_a = sinv_a;
  p.sinv_b = sinv_b;
  p.bias = bias;
  p.out = out_bf16;
  p.out_vec = !out8 && (reinterpret_cast<uintptr_t>(out_bf16) % 16 == 0) && (N % 8 == 0) && (c_stride % 8 == 0);
  p.out8_vec = out8 && (reinterpret_cast<uintptr_t>(ex->out8) % 16 == 0) && (N % 16 == 0) && (c_stride % 16 == 0);
  p.tma_store = out8 ? p.out8_vec : p.out_vec;
  p.bias_vec = bias != nullptr && (reinterpret_cast<uintptr_t>(bias) % 16 == 0);
  const uint32_t fa = (layout & FP8_MM_A_E5M2) ? 1u : 0u;
  const uint32_t fb = (layout & FP8_MM_B_E5M2) ? 1u : 0u;
  // Instruction descriptor: fp32 accumulator (bits 4-5 = 1), A format bits 7-9,
  // B format bits 10-12 (0 = E4M3, 1 = E5M2), A/B major bits 15/16 (1 = MN-major);
  // N/8 (bits 17-22) and M/16 (bits 24-28) are added by the launcher.
  p.a_mn = a_mn;
  p.b_mn = b_mn;
  p.idesc = (1u << 4) | (fa << 7) | (fb << 10) | (a_mn ? 1u << 15 : 0u) | (b_mn ? 1u << 16 : 0u);
  p.err = error_word_ptr();
  return FP8_OK;
}

int launch_bias_only(const MmProblem& q, cudaStream_t st) {
  const int64_t total = q.batch * q.M * q.N;
  const int grid = int(std::min<int64_t>((total + 255) / 256, 4096));
  const cudaError_t e = launch_pdl(mm_bias_only_kernel, dim3(grid), dim3(256), 0, st, 1, q.p, q.M, q.N, q.batch);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

int launch_out8_small(const MmProblem& q, cudaStream_t st) {
  const cudaError_t e = launch_pdl(mm_out8_small_kernel, dim3(1), dim3(256), 0, st, 1, q.p, q.M, q.N, q.batch);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

int mm_run(MmProblem& q, void* workspace, size_t ws_bytes, cudaStream_t st) {
  if ((q.epi & kEpiOut8) && (q.nothing || q.K == 0)) return launch_out8_small(q, st);
  if (q.nothing) return FP8_OK;
  if (q.K == 0) return launch_bias_only(q, st);
  const int sms = sm_count();
  if (sms <= 0) return FP8_ERR_CUDA;
  if (workspace != nullptr && reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return FP8_ERR_UNSUPPORTED;
  const MmChoice c = choose_mm(q.M, q.N, q.K, q.batch, sms, q.p.b_mn, workspace ? ws_bytes : 0);
  if (c.pair == 2) return launch_mm<256, 2>(q.A, q.B, q.M, q.N, q.K, q.batch, q.strides, q.p, q.epi, c, workspace, st);
  if (c.bn == 256) return launch_mm<256, 1>(q.A, q.B, q.M, q.N, q.K, q.batch, q.strides, q.p, q.epi, c, workspace, st);
  if (c.bn == 128) return launch_mm<128, 1>(q.A, q.B, q.M, q.N, q.K, q.batch, q.strides, q.p, q.epi, c, workspace, st);
  return launch_mm<64, 1>(q.A, q.B, q.M, q.N, q.K, q.batch, q.strides, q.p, q.epi, c, workspace, st);
}

}  // namespace
}  // namespace fp8ds

namespace fp8ds {
int mm_args_check(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
                  const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b, const float* bias,
                  const uint16_t* out_bf16) {
  MmProblem q;
  return mm_validate(A, B, M, N, K, batch, strides, layout, sinv_a, sinv_b, bias, const_cast<uint16_t*>(out_bf16), q);
}
}  // namespace fp8ds

static int mm_impl(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
                   const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b, const float* bias,
                   uint16_t* out_bf16, void* workspace, size_t ws_bytes, fp8_stream_t stream) {
  MmProblem q;
  const int rc = mm_validate(A, B, M, N, K, batch, strides, layout, sinv_a, sinv_b, bias, out_bf16, q);
  if (rc != FP8_OK) return rc;
  return mm_run(q, workspace, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int fp8_mm(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
                      const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b,
                      const float* bias, uint16_t* out_bf16, fp8_stream_t stream) {
  return mm_impl(A, B, M, N, K, batch, strides, layout, sinv_a, sinv_b, bias, out_bf16, nullptr, 0, stream);
}

extern "C" int fp8_mm_ws(const uint8_t* A, const uint8_t* B, int64_t M, int64_t N, int64_t K, int64_t batch,
                         const int64_t* strides, int layout, const float* sinv_a, const float* sinv_b,
                         const float* bias, uint16_t* out_bf16, void* workspace, size_t workspace_bytes,
                         fp8_stream_t stream) {
  return mm_impl(A, B, M, N, K, batch, strides, layout, sinv_a, sinv_b, bias, out_bf16, workspace, workspace_bytes,
                 stream);
}

extern "C" int fp8_mm_ex(const fp8_mm_ex_args* a, void* workspace, size_t workspace_bytes, fp8_stream_t stream) {
  if (a == nullptr) return FP8_ERR_INVALID_ARG;
  const bool bias8 = a->bias_scale != nullptr;
  const bool out8 = a->out_kind != FP8_MM_OUT_BF16;
  MmEpilogue ex{bias8 ? static_cast<const uint8_t*>(a->bias) : nullptr, a->bias_scale, a->out_kind,
                out8 ? static_cast<uint8_t*>(a->out) : nullptr, a->out_ring, a->out_amax};
  MmProblem q;
  const int rc = mm_validate(a->A, a->B, a->M, a->N, a->K, a->batch, a->strides, a->layout, a->sinv_a, a->sinv_b,
                             bias8 ? nullptr : static_cast<const float*>(a->bias),
                             out8 ? nullptr : static_cast<uint16_t*>(a->out), q, &ex);
  if (rc != FP8_OK) return rc;
  return mm_run(q, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int fp8_mm_pair(const fp8_mm_args* a0, const fp8_mm_args* a1, void* workspace, size_t workspace_bytes,
                           fp8_stream_t stream) {
  if (a0 == nullptr || a1 == nullptr) return FP8_ERR_INVALID_ARG;
  MmProblem q0, q1;
  int rc = mm_validate(a0->A, a0->B, a0->M, a0->N, a0->K, a0->batch, a0->strides, a0->layout, a0->sinv_a,
                       a0->sinv_b, a0->bias, a0->out_bf16, q0);
  if (rc != FP8_OK) return rc;
  rc = mm_validate(a1->A, a1->B, a1->M, a1->N, a1->K, a1->batch, a1->strides, a1->layout, a1->sinv_a, a1->sinv_b,
                   a1->bias, a1->out_bf16, q1);
  if (rc != FP8_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto separately = [&]() {
    int r = mm_run(q0, workspace, workspace_bytes, st);
    return r != FP8_OK ? r : mm_run(q1, workspace, workspace_bytes, st);
  };
  if (q0.nothing || q1.nothing || q0.K == 0 || q1.K == 0) return separately();
  const int sms = sm_count();
  if (sms <= 0) return FP8_ERR_CUDA;
  if (workspace != nullptr && reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return FP8_ERR_UNSUPPORTED;
  // Shared launch shape: 256-wide tiles, CTA pairs when both problems have
  // more than 128 rows.  CTAs go one at a time to the problem whose whole
  // tiles take longer with the CTAs it has.
  const int pair = (q0.M > kBM && q1.M > kBM) ? 2 : 1;
  const int slots = pair == 2 ? max_pairs<256>(sms) : sms;
  if (slots < 2) return separately();
  const int64_t t0 = ((q0.M + kBM * pair - 1) / (kBM * pair)) * ((q0.N + 255) / 256) * q0.batch;
  const int64_t t1 = ((q1.M + kBM * pair - 1) / (kBM * pair)) * ((q1.N + 255) / 256) * q1.batch;
  const int64_t kb0 = (q0.K + kBK - 1) / kBK, kb1 = (q1.K + kBK - 1) / kBK;
  int64_t c0 = 1, c1 = 1;
  auto span = [](int64_t tiles, int64_t c, int64_t kb) { return ((tiles + c - 1) / c) * kb; };
  while (c0 + c1 < slots) {
    const bool grow0 = c0 < t0 && (span(t0, c0, kb0) >= span(t1, c1, kb1) || c1 >= t1);
    if (grow0) ++c0;
    else if (c1 < t1) ++c1;
    else break;
  }
  // The same time model as choose_mm: one launch's fixed cost, 256-wide tiles.
  const double paired = (pair == 2 ? 5.1 : 4.6) +
                        double(std::max(span(t0, c0, kb0), span(t1, c1, kb1))) * (pair == 2 ? 0.41 : 0.44);
  const size_t wl = workspace ? workspace_bytes : 0;
  const double apart = choose_mm(q0.M, q0.N, q0.K, q0.batch, sms, q0.p.b_mn, wl).cost +
                       choose_mm(q1.M, q1.N, q1.K, q1.batch, sms, q1.p.b_mn, wl).cost;
  if (paired > 0.97 * apart) return separately();
  const MmChoice ch0{256, pair, int(c0), int(t0), 0, 0, 0.0};
  const MmChoice ch1{256, pair, int(c1), int(t1), 0, 0, 0.0};
  return pair == 2 ? launch_pair<256, 2>(q0, ch0, q1, ch1, st) : launch_pair<256, 1>(q0, ch0, q1, ch1, st);
}

extern "C" int fp8_mm_launch_shape(int64_t M, int64_t N, int64_t K, int64_t batch, int layout,
                                   size_t workspace_bytes, int32_t* shape) {
  if (shape == nullptr || M <= 0 || N <= 0 || K <= 0 || batch < 1) return FP8_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return FP8_ERR_CUDA;
  const MmChoice c = choose_mm(M, N, K, batch, sms, (layout & FP8_MM_B_MN_MAJOR) != 0, workspace_bytes);
  shape[0] = c.bn;
  shape[1] = c.pair;
  shape[2] = c.grid * c.pair;
  shape[3] = c.sk_ctas;
  return FP8_OK;
}

extern "C" size_t fp8_mm_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t batch, int layout) {
  if (M <= 0 || N <= 0 || K <= 0 || batch < 1) return 0;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  const MmChoice c = choose_mm(M, N, K, batch, sms, (layout & FP8_MM_B_MN_MAJOR) != 0, size_t(1) << 40);
  return c.ws_bytes;
}
