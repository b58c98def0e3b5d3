// fp8_quantize: delayed-scaling cast of bf16/fp16/fp32 to E4M3/E5M2 on sm_100a.
//
// What is computed follows the AstrAI pages: "tests/extension" (ring commit:
// the last block folds amax into the history window and publishes the next
// scale with an atomic ticket and fences; quantize bindings commit: row /
// transposed / dual QuantLayout), "csrc/kernels/fp8/quantize.cuh" (one tiled
// transpose kernel with vector loads and a scalar fallback for ragged or
// unaligned rows) and "csrc/kernels/fp8_mm.cu" (amax of the raw values).
//
// B200 design (not the pages' sm_89 one):
//   * ROW layout is a flat stream: each thread converts 16 elements per step
//     and writes one 16-byte store; loads are 16-byte vectors, realigned with
//     funnel shifts when the input base is only element-aligned (a 2-byte
//     offset for bf16), so the misaligned case reads HBM at full width too.
//     Grid = one wave of resident blocks, every thread taking the same
//     number of chunks, two in flight at a time.
//   * T / DUAL use a 128x64 tile per 256-thread block: each lane converts a
//     4-row x 8-column patch, packs the 4 rows of each column into one 32-bit
//     word, writes it to a padded shared tile (pitch 33 words: conflict-free
//     writes and reads) and the block streams 128-byte rows of out_t.
//   * amax: fmaxf over |x| (NaN ignored) -> warp shuffle -> block -> one
//     atomic update of the float bits per block (non-negative floats order as
//     unsigned integers), then an acq_rel atomic ticket that orders each
//     block's amax before its increment; the block that draws the last
//     ticket acquires them all, folds the ring, publishes the
//     scale and resets the scratch words to zero for the next call (no
//     memset launch, no host involvement).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "fp8_ring.cuh"

namespace fp8ds {
namespace {

constexpr int kThreads = 256;     // tile, amax and fallback kernels
constexpr int kRowThreads = 256;  // ROW kernel block size
constexpr int kRowMinChunks = 2;  // 16-element chunks per ROW thread, at least

// Three modes: fold (history set, amax_out null), local (amax_out set: the
// last block writes the grid's amax and scale_inv and does not fold; the
// fold follows after a cross-rank MAX of the amax) and fixed scale (both
// null: current scaling's cast pass).
struct RingArgs {
  float* history;
  int32_t* idx;
  float* scale;
  float* scale_inv;
  uint32_t* scratch;
  float* amax_out;
};

// ---- element loads -----------------------------------------------------------

template <int DT> struct In;
template <> struct In<FP8_IN_BF16> { static constexpr int kBytes = 2; };
template <> struct In<FP8_IN_FP16> { static constexpr int kBytes = 2; };
template <> struct In<FP8_IN_FP32> { static constexpr int kBytes = 4; };

template <int DT>
__device__ __forceinline__ float load_one(const uint8_t* p) {
  if constexpr (DT == FP8_IN_BF16) {
    return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t*>(p)) << 16);
  } else if constexpr (DT == FP8_IN_FP16) {
    return __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(p)));
  } else {
    return *reinterpret_cast<const float*>(p);
  }
}

// Two 16-bit elements packed in one word -> floats (low half first).
template <int DT>
__device__ __forceinline__ void unpack2(uint32_t w, float& lo, float& hi) {
  if constexpr (DT == FP8_IN_BF16) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    float2 f = __half22float2(h);
    lo = f.x;
    hi = f.y;
  }
}

__device__ __forceinline__ uint4 ldg16(const uint8_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Words [0, NW) of the byte stream that starts `ph` bytes past the 16-byte
// aligned address `q`, given the aligned words W[0, NW + 4).  ph is a multiple
// of the element size; the word shift is selected without dynamic register
// indexing and the half-word remainder (16-bit types only) is a funnel shift.
template <int NW>
__device__ __forceinline__ void realign(const uint32_t (&W)[NW + 4], int ph, uint32_t (&D)[NW]) {
  const int ws = ph >> 2;
  uint32_t X[NW + 1];
#pragma unroll
  for (int i = 0; i <= NW; ++i) {
    uint32_t a = W[i], b = W[i + 1], c = W[i + 2], d = W[i + 3];
    X[i] = ws == 0 ? a : (ws == 1 ? b : (ws == 2 ? c : d));
  }
  const bool half = (ph & 2) != 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) D[i] = half ? __funnelshift_r(X[i], X[i + 1], 16) : X[i];
}

// Load N (8 or 16) consecutive elements starting at element address p into v.
// Only 16-byte granules that hold at least one of the N elements are read.
template <int DT, int N>
__device__ __forceinline__ void load_vec(const uint8_t* p, float (&v)[N]) {
  constexpr int kB = In<DT>::kBytes;
  constexpr int NW = N * kB / 4;      // useful words
  constexpr int NG = NW / 4;          // useful granules when aligned
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  const int ph = int(a & 15);
  const uint8_t* q = p - ph;
  uint32_t W[NW + 4];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    uint4 t = ldg16(q + 16 * g);
    W[4 * g] = t.x; W[4 * g + 1] = t.y; W[4 * g + 2] = t.z; W[4 * g + 3] = t.w;
  }
  if (ph != 0) {
    uint4 t = ldg16(q + 16 * NG);
    W[4 * NG] = t.x; W[4 * NG + 1] = t.y; W[4 * NG + 2] = t.z; W[4 * NG + 3] = t.w;
  } else {
    W[4 * NG] = W[4 * NG + 1] = W[4 * NG + 2] = W[4 * NG + 3] = 0u;
  }
  uint32_t D[NW];
  realign<NW>(W, ph, D);
  if constexpr (kB == 2) {
#pragma unroll
    for (int i = 0; i < NW; ++i) unpack2<DT>(D[i], v[2 * i], v[2 * i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < NW; ++i) v[i] = __uint_as_float(D[i]);
  }
}

// Aligned fast path (p is 16-byte aligned).
template <int DT, int N>
__device__ __forceinline__ void load_vec_aligned(const uint8_t* p, float (&v)[N]) {
  constexpr int kB = In<DT>::kBytes;
  constexpr int NW = N * kB / 4;
#pragma unroll
  for (int g = 0; g < NW / 4; ++g) {
    uint4 t = ldg16(p + 16 * g);
    uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if constexpr (kB == 2) {
        unpack2<DT>(w[i], v[8 * g + 2 * i], v[8 * g + 2 * i + 1]);
      } else {
        v[4 * g + i] = __uint_as_float(w[i]);
      }
    }
  }
}

// ---- conversion ------------------------------------------------------------

// Running max of |x| over 16-bit pairs: max.xorsign.abs keeps max(|a|, |b|)
// per half (the sign bit of the result is meaningless and masked at the
// end); a NaN operand yields the other operand, as fmaxf does.
template <int DT>
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t w) {
  uint32_t r;
  if constexpr (DT == FP8_IN_BF16)
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w));
  else
    asm("max.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w));
  return r;
}

template <int DT>
__device__ __forceinline__ float absmax2_to_float(uint32_t acc) {
  float lo, hi;
  unpack2<DT>(acc & 0x7FFF7FFFu, lo, hi);
  return fmaxf(lo, hi);
}

// 4x4 byte transpose: word r holds bytes (r, 0..3); output word c holds bytes
// (0..3, c), i.e. byte r of c_out is byte c of r_in.  Eight byte permutes.
__device__ __forceinline__ void transpose4x4(uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3, uint32_t& c0,
                                             uint32_t& c1, uint32_t& c2, uint32_t& c3) {
  const uint32_t t0 = __byte_perm(r0, r1, 0x5140);  // r0.b0 r1.b0 r0.b1 r1.b1
  const uint32_t t1 = __byte_perm(r0, r1, 0x7362);  // r0.b2 r1.b2 r0.b3 r1.b3
  const uint32_t t2 = __byte_perm(r2, r3, 0x5140);
  const uint32_t t3 = __byte_perm(r2, r3, 0x7362);
  c0 = __byte_perm(t0, t2, 0x5410);
  c1 = __byte_perm(t0, t2, 0x7632);
  c2 = __byte_perm(t1, t3, 0x5410);
  c3 = __byte_perm(t1, t3, 0x7632);
}

// ---- amax + ring fold --------------------------------------------------------

// Block-reduce the per-thread amax, publish it with one atomicMax, draw a
// ticket; the last of the `nblocks` blocks working on this ring folds it.
// Must be called by every thread of the block.
// The ring's history and idx are not written until the last block runs, so
// each block reads them early (prefetch_ring at kernel start, one lane per
// word) and the fold itself needs no dependent global reads besides the
// amax word.
struct RingCache {
  float hist;  // history[threadIdx.x] for threads 0..15
  int idx;     // read by thread 16
};

__device__ __forceinline__ RingCache prefetch_ring(const RingArgs& ring) {
  RingCache c{0.0f, 0};
  if (ring.history == nullptr || ring.amax_out != nullptr) return c;  // no fold in this call
  if (threadIdx.x < kHistoryLen) c.hist = ring.history[threadIdx.x];
  if (threadIdx.x == kHistoryLen) c.idx = *ring.idx;
  return c;
}

// Adds a block's amax m (>= 0) to the ring's amax word and draws the block's
// ticket (its arrival number among the blocks on this ring).  No fence: the
// max is an atom that returns only once the word holds the block's amax, and
// the ticket's address is computed from that return (bit 31 of a
// non-negative float's bits: 0 at run time, opaque to the compiler), so the
// ticket cannot be issued before the amax update is performed in L2.  The
// block that draws the last ticket exchanges the amax word only after that
// ticket returned -- after every other block's ticket, hence after every
// other block's amax update, was performed at the same L2 location.  Every
// global atomic a block issued earlier (the TMA producer's tile claims) must
// have returned before the block's final barrier for the same reason.  A
// release-ordered ticket would wait for the block's own output stores to
// complete; without it a 12.6M-element bf16 row quantize takes 8.6 instead of
// 9.0 us on B200.
__device__ __forceinline__ unsigned publish_amax_take_ticket(uint32_t* scratch, float m) {
  uint32_t old, dep, t;
  asm volatile("atom.relaxed.gpu.global.max.u32 %0, [%1], %2;" : "=r"(old) : "l"(scratch), "r"(__float_as_uint(m))
               : "memory");
  asm volatile("shr.u32 %0, %1, 31;" : "=r"(dep) : "r"(old));
  asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], 1;" : "=r"(t) : "l"(scratch + 1 + dep) : "memory");
  return t;
}

template <int FMT, int NT = kThreads>
__device__ __forceinline__ void amax_ticket_fold(float amax, const RingArgs& ring, float s_used,
                                                 const RingCache& rc, const unsigned nblocks) {
  __shared__ float warp_max[NT / 32];
  __shared__ float hist_s[kHistoryLen];
  __shared__ int idx_s;
  __shared__ int last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if (lane == 0) warp_max[warp] = amax;
  if (threadIdx.x < kHistoryLen) hist_s[threadIdx.x] = rc.hist;
  if (threadIdx.x == kHistoryLen) idx_s = rc.idx;
  __syncthreads();
  if (ring.history == nullptr && ring.amax_out == nullptr) {
    // Fixed scale: no amax to publish; the last block clears the scratch
    // words (the tile counter is shared by every kernel that claims tiles).
    if (threadIdx.x == 0) {
      unsigned t;
      asm volatile("atom.relaxed.gpu.global.add.u32 %0, [%1], 1;" : "=r"(t) : "l"(ring.scratch + 1) : "memory");
      if (t == nblocks - 1) {
        asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(ring.scratch + 1) : "memory");
        asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(ring.scratch + 2) : "memory");
      }
    }
    return;
  }
  if (threadIdx.x == 0) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) m = fmaxf(m, warp_max[w]);
    // (A single 64-bit compare-and-swap carrying amax and ticket was tried:
    // hundreds of blocks finishing together made its retries quadratic.)
    const unsigned t = publish_amax_take_ticket(ring.scratch, m);
    last = (t == nblocks - 1);
    if (last) {
      uint32_t bits;
      asm volatile("atom.relaxed.gpu.global.exch.b32 %0, [%1], 0;" : "=r"(bits) : "l"(ring.scratch) : "memory");
      const float a = __uint_as_float(bits);
      asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(ring.scratch + 1) : "memory");
      asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(ring.scratch + 2) : "memory");  // tile counter
      if (ring.amax_out != nullptr) {
        // Local mode: this rank's amax for the cross-rank MAX; the scale the
        // call used is already known, so its inverse is published now.
        *ring.amax_out = a;
        *ring.scale_inv = __frcp_rn(s_used);
        return;
      }
      ring_commit<FMT>(a, hist_s, idx_s, ring.history, ring.idx, ring.scale, ring.scale_inv, s_used);
    }
  }
}

// ---- ROW layout --------------------------------------------------------------

struct RowArgs {
  const uint8_t* in;   // element 0
  uint8_t* out;
  int64_t n;           // elements
  int64_t head;        // scalar elements before the first 16-byte aligned output byte
  int64_t nchunks;     // 16-element chunks after the head
  RingArgs ring;
};

template <int DT, int FMT, bool kAligned>
__device__ __forceinline__ void row_chunk(const RowArgs& a, int64_t j, float s, float& amax) {
  constexpr int kB = In<DT>::kBytes;
  const int64_t e = a.head + 16 * j;
  float v[16];
  if constexpr (kAligned) load_vec_aligned<DT, 16>(a.in + e * kB, v);
  else load_vec<DT, 16>(a.in + e * kB, v);
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = cvt4<FMT>(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3], s);
  *reinterpret_cast<uint4*>(a.out + e) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Block `blk` of the `nblk` blocks that work on tensor a.
template <int DT, int FMT, bool kAligned>
__device__ __forceinline__ void row_body(const RowArgs& a, const unsigned blk, const unsigned nblk) {
  constexpr int kB = In<DT>::kBytes;
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  const float s = *a.ring.scale;
  const RingCache rc = prefetch_ring(a.ring);
  float amax = 0.0f;
  const int64_t tid = int64_t(blk) * kRowThreads + threadIdx.x;
  const int64_t nthr = int64_t(nblk) * kRowThreads;

  // Head and tail (fewer than 16 elements each): one element per thread.
  const int64_t tail0 = a.head + 16 * a.nchunks;
  if (tid < a.head) {
    const float x = load_one<DT>(a.in + tid * kB);
    amax = fmaxf(amax, fabsf(x));
    a.out[tid] = cvt_one<FMT>(x, s);
  }
  if (tid < a.n - tail0) {
    const int64_t e = tail0 + tid;
    const float x = load_one<DT>(a.in + e * kB);
    amax = fmaxf(amax, fabsf(x));
    a.out[e] = cvt_one<FMT>(x, s);
  }

  for (int64_t j = tid; j < a.nchunks; j += 2 * nthr) {
    row_chunk<DT, FMT, kAligned>(a, j, s, amax);
    if (j + nthr < a.nchunks) row_chunk<DT, FMT, kAligned>(a, j + nthr, s, amax);
  }
  amax_ticket_fold<FMT, kRowThreads>(amax, a.ring, s, rc, nblk);
}

template <int DT, int FMT, bool kAligned>
__global__ void __launch_bounds__(kRowThreads) quantize_row_kernel(const __grid_constant__ RowArgs a) {
  row_body<DT, FMT, kAligned>(a, blockIdx.x, gridDim.x);
}

// Several tensors in one launch: blocks [split[s], split[s+1]) cast tensor
// s, each set with its own ring and ticket (one instantiation of the row body
// per format, chosen per block).
constexpr int kMaxMulti = 8;

struct RowMultiArgs {
  RowArgs a[kMaxMulti];
  int fmt[kMaxMulti];
  unsigned split[kMaxMulti + 1];
  int n;
};

template <int DT, bool kAligned>
__global__ void __launch_bounds__(kRowThreads) quantize_row_multi_kernel(const __grid_constant__ RowMultiArgs m) {
  int s = 0;
  while (s + 1 < m.n && blockIdx.x >= m.split[s + 1]) ++s;
  const unsigned blk = blockIdx.x - m.split[s], nblk = m.split[s + 1] - m.split[s];
  if (m.fmt[s] == FP8_E5M2) row_body<DT, FP8_E5M2, kAligned>(m.a[s], blk, nblk);
  else row_body<DT, FP8_E4M3, kAligned>(m.a[s], blk, nblk);
}

// ---- T / DUAL layouts --------------------------------------------------------

constexpr int kTileR = 128;  // input rows per tile
constexpr int kTileC = 64;   // input columns per tile
constexpr int kPitchW = kTileR / 4 + 1;  // shared tile pitch in words (33)

struct TileArgs {
  const uint8_t* in;
  uint8_t* out;     // [rows, cols] (DUAL only)
  uint8_t* out_t;   // [cols, rows]
  int64_t rows, cols;
  int64_t tiles_c, ntiles;
  int out8;         // out rows start 8-byte aligned (base and cols % 8)
  int outt4;        // out_t rows start 4-byte aligned (base and rows % 4)
  RingArgs ring;
};

template <int DT, int FMT, bool kDual>
__global__ void __launch_bounds__(kThreads) quantize_tile_kernel(const TileArgs a) {
  constexpr int kB = In<DT>::kBytes;
  __shared__ uint32_t sT[kTileC * kPitchW];
  // DUAL with rows that are not 8-byte aligned: the tile's row-layout codes,
  // [128 rows][64 bytes], leave as 32-byte coalesced warp stores.
  __shared__ uint2 sR[kDual ? kTileR * kTileC / 8 : 1];
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  const float s = *a.ring.scale;
  const RingCache rc = prefetch_ring(a.ring);
  float amax = 0.0f;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lr0 = 32 * (warp & 3) + 4 * (lane & 7);  // first of this lane's 4 rows
  const int lc0 = 32 * (warp >> 2) + 8 * (lane >> 3);  // first of its 8 columns

  for (int64_t t = blockIdx.x; t < a.ntiles; t += gridDim.x) {
    const int64_t r0 = (t / a.tiles_c) * kTileR;
    const int64_t c0 = (t % a.tiles_c) * kTileC;
    const bool interior = (r0 + kTileR <= a.rows) && (c0 + kTileC <= a.cols);
    uint32_t q[4][2];  // 4 rows x 8 codes
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t r = r0 + lr0 + i;
      const int64_t c = c0 + lc0;
      float v[8];
      if (interior) {
        load_vec<DT, 8>(a.in + (r * a.cols + c) * kB, v);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          v[j] = (r < a.rows && c + j < a.cols) ? load_one<DT>(a.in + (r * a.cols + c + j) * kB) : 0.0f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
      q[i][0] = cvt4<FMT>(v[0], v[1], v[2], v[3], s);
      q[i][1] = cvt4<FMT>(v[4], v[5], v[6], v[7], s);
      if constexpr (kDual) {
        if (a.out8) {
          uint8_t* o = a.out + r * a.cols + c;
          if (interior) {
            *reinterpret_cast<uint2*>(o) = make_uint2(q[i][0], q[i][1]);
          } else if (r < a.rows) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              if (c + j < a.cols) o[j] = uint8_t(q[i][j >> 2] >> (8 * (j & 3)));
          }
        }
      }
    }
    __syncthreads();  // previous tile's readers are done with sT and sR
    if constexpr (kDual) {
      if (!a.out8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) sR[(lr0 + i) * (kTileC / 8) + (lc0 >> 3)] = make_uint2(q[i][0], q[i][1]);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t c[4];
      transpose4x4(q[0][h], q[1][h], q[2][h], q[3][h], c[0], c[1], c[2], c[3]);
#pragma unroll
      for (int k = 0; k < 4; ++k) sT[(lc0 + 4 * h + k) * kPitchW + (lr0 >> 2)] = c[k];
    }
    __syncthreads();
    if constexpr (kDual) {
      if (!a.out8) {
        // Warp w writes rows 16w .. 16w+15 of the tile, lane l bytes l and l+32.
        const uint8_t* sRb = reinterpret_cast<const uint8_t*>(sR);
#pragma unroll 4
        for (int k = 0; k < kTileR / 8; ++k) {
          const int rl = (kTileR / 8) * warp + k;
          const int64_t r = r0 + rl;
          if (r < a.rows) {
            uint8_t* o = a.out + r * a.cols + c0;
            if (c0 + lane < a.cols) o[lane] = sRb[rl * kTileC + lane];
            if (c0 + lane + 32 < a.cols) o[lane + 32] = sRb[rl * kTileC + lane + 32];
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kTileC / 8; ++k) {
      const int cl = 8 * warp + k;
      const int64_t c = c0 + cl;
      const int64_t r = r0 + 4 * lane;
      const uint32_t w = sT[cl * kPitchW + lane];
      if (c < a.cols) {
        uint8_t* o = a.out_t + c * a.rows + r;
        if (a.outt4 && r + 4 <= a.rows) {
          *reinterpret_cast<uint32_t*>(o) = w;
        } else {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            if (r + b < a.rows) o[b] = uint8_t(w >> (8 * b));
        }
      }
    }
  }
  amax_ticket_fold<FMT>(amax, a.ring, s, rc, gridDim.x);
}

// ---- T / DUAL layouts, warp-specialised TMA pipeline (16-byte aligned rows) -------
//
// Same 128x64 tiles and lane mapping as quantize_tile_kernel.  Warp 8 is the
// producer: it claims tiles from a counter in the ring's scratch (so blocks
// that finish early take more tiles and all blocks end within one tile of
// each other), writes the tile id into shared memory and loads the tile with
// TMA (128 rows x 128 bytes per box, 128B-swizzled) into a kStages-deep ring.
// Warps 0..7 consume: each warp releases a stage with one mbarrier arrive as
// soon as its lanes have read it, converts, writes the DUAL row pieces, and
// transposes into one of two 8 KB buffers (16-byte units XOR-swizzled by the
// column group); one named-barrier reduction per tile publishes the buffer
// and makes the stop decision uniform, and the buffer leaves as 16-byte
// stores of 128-byte out_t rows.  Ragged edges are zero-filled by TMA and the
// stores are guarded.  Used when the input base is 16-byte aligned and a row
// is a multiple of 16 bytes.

constexpr int kConsumerWarps = 8;
constexpr int kWsThreads = 32 * (kConsumerWarps + 1);
constexpr uint32_t kNoTile = 0xFFFFFFFFu;

// kShift: an input base that is only element-aligned, rows a multiple of 16
// bytes (see tile_tma_body): each tile row is staged as 64 + 16 / in_bytes
// elements (the tile's columns plus the slack of rounding the box start down
// to 16 bytes), unswizzled.
template <int DT, bool kShift = false>
struct TmaTile {
  static constexpr int kBoxes = In<DT>::kBytes == 4 ? 2 : 1;  // 128-byte-wide boxes per 64-column tile
  static constexpr int kBoxBytes = kTileR * 128;
  static constexpr int kSRowBytes = (kTileC + 16 / In<DT>::kBytes) * In<DT>::kBytes;  // 144 / 272
  static constexpr int kStageBytes = kShift ? kTileR * kSRowBytes : kBoxes * kBoxBytes;
  static constexpr int kStages = DT == FP8_IN_FP32 ? 2 : 3;
  static constexpr int kTBytes = kTileC * kTileR;  // one transpose buffer: 64 rows of 128 bytes
  static constexpr int kBarOff = kStages * kStageBytes + 2 * kTBytes;
  static constexpr int kSmem = kBarOff + 16 * kStages + 8 * kStages + 64 + 1024;
};

struct TmaTileArgs {
  TileArgs t;
  uint32_t* err;
  unsigned long long wait_ns;  // budget of the producer's and consumers' waits on each other
  uint32_t stall;              // kWaitQuantizeTma: consumers wait on a never-completed barrier (testing)
  // kShift only: the map starts off_e elements before the input base (at the
  // base rounded down to 16 bytes), so input column c is map column off_e + c.
  int off_e;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool bar_try_wait(uint32_t bar, uint32_t parity) {
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

__device__ __forceinline__ bool bar_wait_bounded(uint32_t bar, uint32_t parity,
                                                 unsigned long long budget_ns = kWaitBudgetNs) {
  if (bar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!bar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > budget_ns) return false;
  }
  return true;
}

__device__ __forceinline__ void bar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// mbarrier arrive issued only once `dep` is available: the predicate that
// guards it is computed from dep, and no value of dep makes it false.
__device__ __forceinline__ void bar_arrive_after(uint32_t bar, uint32_t dep) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 d;\n\t"
      "and.b32 d, %1, 0x7FFFFFFF;\n\t"
      "setp.ne.u32 p, d, 0xFFFFFFFF;\n\t"
      "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(bar), "r"(dep)
      : "memory");
}

// OR-reduction barrier over the consumer warps only (named barrier 1).
__device__ __forceinline__ bool consumers_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u), "r"(32 * kConsumerWarps)
      : "memory");
  return r != 0;
}

template <int DT>
__device__ __forceinline__ void issue_tile_load(const CUtensorMap* tm, uint32_t dst, uint32_t bar, uint32_t t,
                                                uint32_t tiles_c) {
  const uint32_t tr = t / tiles_c;
  const int r0 = int(tr * kTileR);
  const int c0 = int((t - tr * tiles_c) * kTileC);
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(uint32_t(TmaTile<DT>::kStageBytes))
               : "memory");
#pragma unroll
  for (int bx = 0; bx < TmaTile<DT>::kBoxes; ++bx) {
    const int cx = c0 + bx * (128 / In<DT>::kBytes);
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst + uint32_t(bx * TmaTile<DT>::kBoxBytes)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(cx), "r"(r0), "r"(bar)
        : "memory");
  }
}

// Shifted base: the tile's box starts at map column off_e + c0 rounded down
// to 16 bytes and is 64 + 16 / in_bytes columns wide, so it holds the tile's
// 64 columns whatever the base's offset inside its 16-byte granule.
template <int DT>
__device__ __forceinline__ void issue_tile_load_shift(const CUtensorMap* tm, uint32_t dst, uint32_t bar, uint32_t t,
                                                      uint32_t tiles_c, int off_e) {
  constexpr int kAlign = 16 / In<DT>::kBytes;
  const uint32_t tr = t / tiles_c;
  const int r0 = int(tr * kTileR);
  const int x = (off_e + int(t - tr * tiles_c) * kTileC) & ~(kAlign - 1);
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(uint32_t(TmaTile<DT, true>::kStageBytes))
               : "memory");
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(r0), "r"(bar)
      : "memory");
}

// Eight bytes (lo, hi) to an address of any alignment with the widest
// aligned stores it allows.
__device__ __forceinline__ void store8_any(uint8_t* o, uint32_t lo, uint32_t hi) {
  const int m = int(reinterpret_cast<uintptr_t>(o) & 7);
  if (m == 0) {
    *reinterpret_cast<uint2*>(o) = make_uint2(lo, hi);
  } else if (m == 4) {
    reinterpret_cast<uint32_t*>(o)[0] = lo;
    reinterpret_cast<uint32_t*>(o)[1] = hi;
  } else if ((m & 1) == 0) {
    uint16_t* h = reinterpret_cast<uint16_t*>(o);
    h[0] = uint16_t(lo);
    h[1] = uint16_t(lo >> 16);
    h[2] = uint16_t(hi);
    h[3] = uint16_t(hi >> 16);
  } else {
    o[0] = uint8_t(lo);
    uint16_t* h = reinterpret_cast<uint16_t*>(o + 1);
    h[0] = uint16_t(__byte_perm(lo, 0, 0x0021));
    h[1] = uint16_t(__byte_perm(lo, hi, 0x0043));
    h[2] = uint16_t(__byte_perm(hi, 0, 0x0021));
    o[7] = uint8_t(hi >> 24);
  }
}

// Byte offset of 16-byte unit v of transpose-buffer row c (rows of 128 bytes;
// the unit index is XOR-swizzled by the column group so that the column-word
// writes and the row reads are both free of bank conflicts).
__device__ __forceinline__ int tbuf_unit(int c, int v) { return c * 128 + ((v ^ ((c >> 2) & 6)) << 4); }

template <int DT, int FMT, bool kDual, bool kShift = false>
__device__ __forceinline__ void tile_tma_body(const CUtensorMap* tmIn, const TmaTileArgs& args, const unsigned blk,
                                              const unsigned nblk) {
  using TT = TmaTile<DT, kShift>;
  constexpr int kB = In<DT>::kBytes;
  constexpr int S = TT::kStages;
  const TileArgs& a = args.t;
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* smem = qsmem_raw + ((1024u - (smem_addr(qsmem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  uint8_t* tbuf = smem + S * TT::kStageBytes;
  const uint32_t full0 = sbase + TT::kBarOff;        // full[S]
  const uint32_t empty0 = full0 + 8u * S;            // empty[S]
  volatile uint32_t* tile_id = reinterpret_cast<volatile uint32_t*>(smem + TT::kBarOff + 16 * S);
  const uint32_t stall_bar = full0 + 24u * S;  // after the tile ids: never arrived on

  pdl_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8u * i) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8u * i), "r"(kConsumerWarps) : "memory");
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(stall_bar) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmIn)) : "memory");
  }
  __syncthreads();
  pdl_wait_prior_grid();
  const float s = *a.ring.scale;
  const RingCache rc = prefetch_ring(a.ring);
  float amax = 0.0f;
  const uint32_t tiles_c = uint32_t(a.tiles_c), ntiles = uint32_t(a.ntiles);

  if (warp == kConsumerWarps) {
    // ---------------- producer: claim, then load ----------------
    if (lane == 0) {
      uint32_t armed = 0, armed_par = 0;
      int stage = 0;
      uint32_t phase = 0;
      // The first `rounds` tiles of this block are static (blk, blk + nblk,
      // ..., one per stage, so the ring fills at once); every later tile is
      // claimed from the counter in the ring's scratch, so blocks that run
      // ahead take more (CTAs progress at unequal rates: a static deal of
      // all tiles made a 67M-element DUAL call 20% slower).  Two claims are
      // kept in flight, the first issued two tiles before it is needed.
      // When the static tiles cover the tensor (ntiles <= S * nblk, e.g. a
      // 1536x1536 weight) nothing is claimed: a claim's round trip to L2
      // delayed the static loads that follow it (1536x1536 bf16 T: 6.6 ->
      // 6.0 us without claims on B200).  Issuing all static tiles before
      // any claim was measured too: faster for fp32 (two stages) but 1.4 us
      // slower for 12.6M-element bf16 T, where the three rounds requested
      // at once are 87% of the input and every block's first tile lands late.
      uint32_t* ctr = a.ring.scratch + 2;
      const uint32_t rounds = min(uint32_t(S), (ntiles + nblk - 1) / nblk);
      const uint32_t dyn0 = rounds * nblk;
      const bool dyn = dyn0 < ntiles;
      uint32_t c0 = 0, c1 = 0;  // claims in flight (c0 the older), valid from iteration rounds - 2 on
      for (uint32_t k = 0;; ++k) {
        if (!bar_wait_bounded(empty0 + 8u * stage, phase ^ 1u, args.wait_ns)) {
          record_device_error(args.err, kWaitQuantizeTma);
          break;
        }
        // Claims are issued in program order (so c0 < c1 < later ones): the
        // first two during the last two static tiles, then one per tile.
        uint32_t t;
        if (k < rounds) {
          t = blk + k * nblk;
          if (dyn && k + 2 == rounds) c0 = atomicAdd(ctr, 1u);
          if (dyn && k + 1 == rounds) {
            if (rounds == 1) c0 = atomicAdd(ctr, 1u);
            c1 = atomicAdd(ctr, 1u);
          }
        } else if (dyn) {
          t = dyn0 + c0;
          c0 = c1;
          c1 = atomicAdd(ctr, 1u);
        } else {
          t = kNoTile;
        }
        if (t < ntiles) {
          tile_id[stage] = t;
          if constexpr (kShift)
            issue_tile_load_shift<DT>(tmIn, sbase + uint32_t(stage * TT::kStageBytes), full0 + 8u * stage, t, tiles_c,
                                      args.off_e);
          else
            issue_tile_load<DT>(tmIn, sbase + uint32_t(stage * TT::kStageBytes), full0 + 8u * stage, t, tiles_c);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        } else {
          // The copy last armed on this stage was consumed (its empty phase
          // completed above); the stop marker completes a further phase with
          // no copy, so this stage has nothing left to drain.
          armed &= ~(1u << stage);
          tile_id[stage] = kNoTile;
          bar_arrive_local(full0 + 8u * stage);  // wakes the consumers with the stop marker
          break;
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // Every armed copy has landed before shared memory can be released.
      for (int i = 0; i < S; ++i)
        if (armed & (1u << i)) bar_wait_bounded(full0 + 8u * i, (armed_par >> i) & 1u);
      // The claims still in flight have returned (been performed) before
      // the block's ticket, so the last block's reset of the counter comes
      // after every claim.  (The counter never reaches 0xFFFFFFFF.)
      if ((c0 & c1) == 0xFFFFFFFFu) record_device_error(args.err, kWaitQuantizeTma);
    }
    __syncwarp();
  } else {
    // ---------------- consumers ----------------
    const int lr0 = 32 * (warp & 3) + 4 * (lane & 7);  // first of this lane's 4 rows
    const int lc0 = 32 * (warp >> 2) + 8 * (lane >> 3);  // first of its 8 columns
    const bool out16 = a.outt4 && (a.rows % 16 == 0) && (reinterpret_cast<uintptr_t>(a.out_t) % 16 == 0);
    uint32_t amax2 = 0u;  // packed |x| maxima of 16-bit inputs
    int stage = 0, buf = 0;
    uint32_t phase = 0;
    // (Testing: with the stall site set, the consumers wait on a barrier that
    // nothing completes, so the wait runs out and the kernel stops early.)
    const bool stall = args.stall == kWaitQuantizeTma;
    while (true) {
      const bool ok = bar_wait_bounded(stall ? stall_bar : full0 + 8u * stage, stall ? 0u : phase, args.wait_ns);
      if (!ok) record_device_error(args.err, kWaitQuantizeTma);
      const uint32_t t = ok ? uint32_t(tile_id[stage]) : uint32_t(kNoTile);
      const bool stop = t == kNoTile;
      uint32_t q[4][2];
      if (!stop) {
        const uint8_t* st = smem + stage * TT::kStageBytes;
        if constexpr (kShift) {
          // Staged row rl holds input row r0 + rl from column c0 - d on, where
          // d = (off_e + c0) mod (16 / in_bytes); elements past the last column
          // (zero-filled or the next row's) are set to zero before the amax.
          // Rows 4 apart are 576 bytes apart, so a quarter-warp's loads split
          // over two 64-byte halves of the banks (4-way conflicts).
          constexpr int kAlign = 16 / kB;
          const uint32_t tr = t / tiles_c;
          const int64_t gc = int64_t(t - tr * tiles_c) * kTileC + lc0;  // this lane's first column
          const int d = int((args.off_e + gc - lc0) & (kAlign - 1));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int off = (lr0 + i) * TT::kSRowBytes + (d + lc0) * kB;
            const uint8_t* g16 = st + (off & ~15);
            const int ph = off & 15;
            float v[8];
            if constexpr (kB == 2) {
              uint32_t W[8], D[4];
              const uint4 w0 = *reinterpret_cast<const uint4*>(g16);
              const uint4 w1 = *reinterpret_cast<const uint4*>(g16 + 16);
              W[0] = w0.x; W[1] = w0.y; W[2] = w0.z; W[3] = w0.w;
              W[4] = w1.x; W[5] = w1.y; W[6] = w1.z; W[7] = w1.w;
              realign<4>(W, ph, D);
#pragma unroll
              for (int e = 0; e < 4; ++e) unpack2<DT>(D[e], v[2 * e], v[2 * e + 1]);
            } else {
              uint32_t W[12], D[8];
              const uint4 w0 = *reinterpret_cast<const uint4*>(g16);
              const uint4 w1 = *reinterpret_cast<const uint4*>(g16 + 16);
              const uint4 w2 = ph != 0 ? *reinterpret_cast<const uint4*>(g16 + 32) : make_uint4(0u, 0u, 0u, 0u);
              W[0] = w0.x; W[1] = w0.y; W[2] = w0.z; W[3] = w0.w;
              W[4] = w1.x; W[5] = w1.y; W[6] = w1.z; W[7] = w1.w;
              W[8] = w2.x; W[9] = w2.y; W[10] = w2.z; W[11] = w2.w;
              realign<8>(W, ph, D);
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(D[e]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              if (gc + e >= a.cols) v[e] = 0.0f;
              amax = fmaxf(amax, fabsf(v[e]));
            }
            q[i][0] = cvt4<FMT>(v[0], v[1], v[2], v[3], s);
            q[i][1] = cvt4<FMT>(v[4], v[5], v[6], v[7], s);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = lr0 + i;
            float v[8];
            if constexpr (kB == 2) {
              const int chunk = (lc0 >> 3) ^ (r & 7);
              const uint4 w = *reinterpret_cast<const uint4*>(st + r * 128 + chunk * 16);
              amax2 = absmax2<DT>(absmax2<DT>(amax2, w.x), absmax2<DT>(w.y, absmax2<DT>(w.z, w.w)));
              unpack2<DT>(w.x, v[0], v[1]);
              unpack2<DT>(w.y, v[2], v[3]);
              unpack2<DT>(w.z, v[4], v[5]);
              unpack2<DT>(w.w, v[6], v[7]);
            } else {
              const int box = lc0 >> 5;
              const int ch = (lc0 & 31) >> 2;
              const uint8_t* rowp = st + box * TT::kBoxBytes + r * 128;
              const float4 f0 = *reinterpret_cast<const float4*>(rowp + ((ch ^ (r & 7)) * 16));
              const float4 f1 = *reinterpret_cast<const float4*>(rowp + (((ch + 1) ^ (r & 7)) * 16));
              v[0] = f0.x; v[1] = f0.y; v[2] = f0.z; v[3] = f0.w;
              v[4] = f1.x; v[5] = f1.y; v[6] = f1.z; v[7] = f1.w;
#pragma unroll
              for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(v[j]));
            }
            q[i][0] = cvt4<FMT>(v[0], v[1], v[2], v[3], s);
            q[i][1] = cvt4<FMT>(v[4], v[5], v[6], v[7], s);
          }
        }
      }
      // This warp is done reading the stage: let the producer refill it.
      // Every loaded value went into the amax, and the release is predicated
      // on the warp-wide OR of the lanes' maxima, so no lane's shared-memory
      // load can still be in flight when the next copy lands in the stage.
      {
        const uint32_t dep = __reduce_or_sync(0xFFFFFFFFu, amax2 | __float_as_uint(amax));
        if (lane == 0) bar_arrive_after(empty0 + 8u * stage, dep);
      }
      int64_t r0 = 0, c0 = 0;
      if (!stop) {
        const uint32_t tr = t / tiles_c;
        r0 = int64_t(tr) * kTileR;
        c0 = int64_t(t - tr * tiles_c) * kTileC;
        const bool interior = (r0 + kTileR <= a.rows) && (c0 + kTileC <= a.cols);
        if constexpr (kDual) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int64_t r = r0 + lr0 + i;
            const int64_t c = c0 + lc0;
            uint8_t* o = a.out + r * a.cols + c;
            if (interior && a.out8) {
              *reinterpret_cast<uint2*>(o) = make_uint2(q[i][0], q[i][1]);
            } else if (interior) {
              store8_any(o, q[i][0], q[i][1]);
            } else if (r < a.rows) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (c + j < a.cols) o[j] = uint8_t(q[i][j >> 2] >> (8 * (j & 3)));
            }
          }
        }
        uint8_t* tb = tbuf + buf * TT::kTBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t c[4];
          transpose4x4(q[0][h], q[1][h], q[2][h], q[3][h], c[0], c[1], c[2], c[3]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int col = lc0 + 4 * h + k;
            const int word = lr0 >> 2;  // 4 rows per word
            *reinterpret_cast<uint32_t*>(tb + tbuf_unit(col, word >> 2) + ((word & 3) << 2)) = c[k];
          }
        }
      }
      if (consumers_sync_or(stop)) break;
      // out_t rows: thread -> (column c, 16-byte unit v), two columns per thread.
      {
        const uint8_t* tb = tbuf + buf * TT::kTBytes;
        const int tid = threadIdx.x;  // 0..255
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int col = (tid >> 3) + 32 * i;
          const int v = tid & 7;
          const uint4 w = *reinterpret_cast<const uint4*>(tb + tbuf_unit(col, v));
          const int64_t c = c0 + col;
          const int64_t r = r0 + 16 * v;
          if (c < a.cols) {
            uint8_t* o = a.out_t + c * a.rows + r;
            if (out16 && r + 16 <= a.rows) {
              *reinterpret_cast<uint4*>(o) = w;
            } else {
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int b = 0; b < 16; ++b)
                if (r + b < a.rows) o[b] = uint8_t(ww[b >> 2] >> (8 * (b & 3)));
            }
          }
        }
      }
      buf ^= 1;
      if (++stage == S) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if constexpr (kB == 2) amax = fmaxf(amax, absmax2_to_float<DT>(amax2));
  }
  __syncthreads();
  amax_ticket_fold<FMT, kWsThreads>(amax, a.ring, s, rc, nblk);
}

template <int DT, int FMT, bool kDual, bool kShift = false>
__global__ void __launch_bounds__(kWsThreads) quantize_tile_tma_kernel(const __grid_constant__ CUtensorMap tmIn,
                                                                        const __grid_constant__ TmaTileArgs args) {
  tile_tma_body<DT, FMT, kDual, kShift>(&tmIn, args, blockIdx.x, gridDim.x);
}

// Several tensors in one launch (a linear's X, W and G): blocks
// [split[s], split[s+1]) work on tensor s, each set with its own ring, amax
// ticket and tile counter, so each tensor's result is exactly that of its
// own launch.  The tensors share the dtype and layout (one instantiation of
// the tile body per format, chosen per block).

struct TmaMultiArgs {
  CUtensorMap maps[kMaxMulti];
  TmaTileArgs a[kMaxMulti];
  int fmt[kMaxMulti];
  unsigned split[kMaxMulti + 1];
  int n;
};

template <int DT, bool kDual>
__global__ void __launch_bounds__(kWsThreads) quantize_tile_tma_multi_kernel(const __grid_constant__ TmaMultiArgs m) {
  int s = 0;
  while (s + 1 < m.n && blockIdx.x >= m.split[s + 1]) ++s;
  const unsigned blk = blockIdx.x - m.split[s], nblk = m.split[s + 1] - m.split[s];
  if (m.fmt[s] == FP8_E5M2) tile_tma_body<DT, FP8_E5M2, kDual>(&m.maps[s], m.a[s], blk, nblk);
  else tile_tma_body<DT, FP8_E4M3, kDual>(&m.maps[s], m.a[s], blk, nblk);
}

// ---- current scaling: amax pass ---------------------------------------------------
//
// Current (dynamic) scaling measures the scale from the tensor itself: this
// pass reduces amax exactly as the quantize kernels do (16-byte loads, warp
// shuffle, one relaxed atomic max per block, acq_rel ticket), and the block
// that takes the last ticket publishes scale = FP8_MAX / amax (1 when amax is
// zero or the quotient is not finite), scale_inv = 1 / scale and amax, then
// clears the scratch words.  The cast pass that follows reads that scale.

struct AmaxArgs {
  const uint8_t* in;
  int64_t n, head, nchunks;  // head: scalar elements before the first 16-byte aligned input chunk
  uint32_t* scratch;
  float* scale;
  float* scale_inv;
  float* amax_out;
};

template <int DT, int FMT>
__global__ void __launch_bounds__(kThreads) amax_kernel(const AmaxArgs a) {
  constexpr int kB = In<DT>::kBytes;
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  float amax = 0.0f;
  const int64_t tid = int64_t(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t nthr = int64_t(gridDim.x) * kThreads;
  const int64_t tail0 = a.head + 16 * a.nchunks;
  if (tid < a.head) amax = fmaxf(amax, fabsf(load_one<DT>(a.in + tid * kB)));
  if (tid < a.n - tail0) amax = fmaxf(amax, fabsf(load_one<DT>(a.in + (tail0 + tid) * kB)));
  for (int64_t j = tid; j < a.nchunks; j += 2 * nthr) {
    float v[16], w[16];
    const bool two = j + nthr < a.nchunks;
    load_vec_aligned<DT, 16>(a.in + (a.head + 16 * j) * kB, v);
    if (two) load_vec_aligned<DT, 16>(a.in + (a.head + 16 * (j + nthr)) * kB, w);
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    if (two) {
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(w[i]));
    }
  }
  __shared__ float warp_max[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, warp_max[w]);
    const unsigned t = publish_amax_take_ticket(a.scratch, m);
    if (t == gridDim.x - 1) {
      uint32_t bits;
      asm volatile("atom.relaxed.gpu.global.exch.b32 %0, [%1], 0;" : "=r"(bits) : "l"(a.scratch) : "memory");
      asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(a.scratch + 1) : "memory");
      const float am = __uint_as_float(bits);
      const float fmax = FMT == FP8_E4M3 ? kE4M3Max : kE5M2Max;
      float sc = 1.0f;
      if (am > 0.0f && isfinite(am)) {
        const float c = __fdiv_rn(fmax, am);
        if (isfinite(c) && c > 0.0f) sc = c;
      }
      *a.scale = sc;
      *a.scale_inv = __frcp_rn(sc);
      if (a.amax_out) *a.amax_out = am;
    }
  }
}

// ---- host side ---------------------------------------------------------------

int sm_count_current() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev < 0 || dev >= 64) return -1;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cached[dev] = n;
  }
  return cached[dev];
}

// Resident blocks per SM of a kernel without dynamic shared memory (cached
// per device by the caller's static array).
template <typename Kern>
int resident_blocks(Kern kern, int threads, int (&cached)[64]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, 0) != cudaSuccess || n < 1) return -1;
    cached[dev] = n;
  }
  return cached[dev];
}

// ROW grid: one wave of resident blocks at most, and every thread takes the
// same number of 16-element chunks (at least kRowMinChunks), so no fraction
// of the blocks runs one more round than the rest.
template <int DT, int FMT, bool kAligned>
int launch_row1(const RowArgs& a, int sms, cudaStream_t st) {
  static int cached[64] = {0};
  const int bps = resident_blocks(quantize_row_kernel<DT, FMT, kAligned>, kRowThreads, cached);
  if (bps <= 0) return FP8_ERR_CUDA;
  const int64_t tmax = int64_t(bps) * sms * kRowThreads;
  const int64_t per = std::max<int64_t>(kRowMinChunks, (a.nchunks + tmax - 1) / tmax);
  const int grid = int(std::max<int64_t>(1, (a.nchunks + per * kRowThreads - 1) / (per * kRowThreads)));
  const cudaError_t e = launch_pdl(quantize_row_kernel<DT, FMT, kAligned>, grid, kRowThreads, 0, st, 1, a);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

template <int DT, int FMT>
int launch_row(const RowArgs& a, int sms, cudaStream_t st, bool aligned) {
  return aligned ? launch_row1<DT, FMT, true>(a, sms, st) : launch_row1<DT, FMT, false>(a, sms, st);
}

// Element-aligned T / DUAL tiles: a grid of resident blocks (one wave).
template <int DT, int FMT, bool kDual>
int launch_tile1(const TileArgs& a, int sms, cudaStream_t st) {
  static int cached[64] = {0};
  const int bps = resident_blocks(quantize_tile_kernel<DT, FMT, kDual>, kThreads, cached);
  if (bps <= 0) return FP8_ERR_CUDA;
  const int grid = int(std::max<int64_t>(1, std::min<int64_t>(a.ntiles, int64_t(bps) * sms)));
  const cudaError_t e = launch_pdl(quantize_tile_kernel<DT, FMT, kDual>, grid, kThreads, 0, st, 1, a);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

template <int DT, int FMT>
int launch_tile(const TileArgs& a, int sms, cudaStream_t st, bool dual) {
  return dual ? launch_tile1<DT, FMT, true>(a, sms, st) : launch_tile1<DT, FMT, false>(a, sms, st);
}

template <int DT>
int dispatch_fmt_row(int fmt, const RowArgs& a, int sms, cudaStream_t st, bool aligned) {
  return fmt == FP8_E4M3 ? launch_row<DT, FP8_E4M3>(a, sms, st, aligned)
                         : launch_row<DT, FP8_E5M2>(a, sms, st, aligned);
}

template <int DT>
int dispatch_fmt_tile(int fmt, const TileArgs& a, int sms, cudaStream_t st, bool dual) {
  return fmt == FP8_E4M3 ? launch_tile<DT, FP8_E4M3>(a, sms, st, dual)
                         : launch_tile<DT, FP8_E5M2>(a, sms, st, dual);
}

// 2-D map over the input [rows, cols] with a 128-row x 128-byte box, 128B swizzle.
bool make_input_map(CUtensorMap* m, const void* in, int dtype, int64_t rows, int64_t cols) {
  const int eb = dtype == FP8_IN_FP32 ? 4 : 2;
  const uint64_t dims[2] = {uint64_t(cols), uint64_t(rows)};
  const uint64_t strides[1] = {uint64_t(cols * eb)};
  const uint32_t box[2] = {uint32_t(128 / eb), uint32_t(kTileR)};
  return encode_tiled_cached(m, eb == 4 ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, in,
                             dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// Shifted-base 2-D map: rows a multiple of 16 bytes but an input base that
// is only element-aligned.  The map starts at the base rounded down to 16
// bytes (off_e elements earlier, inside the same 16-byte granule) and its rows
// are cols + off_e elements long, so it ends where the tensor ends.  Boxes are
// 64 + 16 / in_bytes elements by 128 rows, unswizzled.  (Rows that are not a
// multiple of 16 bytes were tried through a map whose rows are g consecutive
// input rows: slower than the register tile kernel at 8192x1537.)
bool make_shifted_map(CUtensorMap* m, const void* in, int dtype, int64_t rows, int64_t cols, int off_e) {
  const int eb = dtype == FP8_IN_FP32 ? 4 : 2;
  const uint8_t* base = static_cast<const uint8_t*>(in) - off_e * eb;
  const uint64_t dims[2] = {uint64_t(cols + off_e), uint64_t(rows)};
  const uint64_t strides[1] = {uint64_t(cols * eb)};
  const uint32_t box[2] = {uint32_t(kTileC + 16 / eb), uint32_t(kTileR)};
  return encode_tiled_cached(m, eb == 4 ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base,
                             dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// Resident blocks per SM of a TMA tile kernel instantiation (cached per device).
template <int DT, int FMT, bool kDual, bool kShift>
int tma_blocks_per_sm() {
  static int cached[64] = {0};
  constexpr int kSmem = TmaTile<DT, kShift>::kSmem;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (cached[dev] == 0) {
    auto kern = quantize_tile_tma_kernel<DT, FMT, kDual, kShift>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) return -1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kWsThreads, kSmem) != cudaSuccess || n < 1) return -1;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int DT, int FMT, bool kDual, bool kShift>
int launch_tile_tma1(const TileArgs& t, const CUtensorMap& map, int off_e, int sms, cudaStream_t st) {
  const WaitCfg wc = wait_cfg();
  TmaTileArgs a{t, error_word_ptr(), wc.budget_ns, wc.stall_site, off_e};
  const int bps = tma_blocks_per_sm<DT, FMT, kDual, kShift>();
  if (bps <= 0) return FP8_ERR_CUDA;
  const int grid = int(std::max<int64_t>(1, std::min<int64_t>(t.ntiles, int64_t(bps) * sms)));
  const cudaError_t e = launch_pdl(quantize_tile_tma_kernel<DT, FMT, kDual, kShift>, grid, kWsThreads,
                                   TmaTile<DT, kShift>::kSmem, st, 1, map, a);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// off_e < 0: the 16-byte aligned kernel; otherwise the shifted-base kernel.
template <int DT, int FMT>
int launch_tile_tma(const TileArgs& t, const CUtensorMap& map, int off_e, int sms, cudaStream_t st, bool dual) {
  if (off_e >= 0)
    return dual ? launch_tile_tma1<DT, FMT, true, true>(t, map, off_e, sms, st)
                : launch_tile_tma1<DT, FMT, false, true>(t, map, off_e, sms, st);
  return dual ? launch_tile_tma1<DT, FMT, true, false>(t, map, 0, sms, st)
              : launch_tile_tma1<DT, FMT, false, false>(t, map, 0, sms, st);
}

template <int DT>
int dispatch_fmt_tile_tma(int fmt, const TileArgs& a, const CUtensorMap& map, int off_e, int sms, cudaStream_t st,
                          bool dual) {
  return fmt == FP8_E4M3 ? launch_tile_tma<DT, FP8_E4M3>(a, map, off_e, sms, st, dual)
                         : launch_tile_tma<DT, FP8_E5M2>(a, map, off_e, sms, st, dual);
}

}  // namespace
}  // namespace fp8ds

using namespace fp8ds;

namespace fp8ds {
namespace {
// Launches the cast kernel for the layout (and the ring fold unless r.history
// is null).  Arguments are already validated.
// One quantize call resolved to its kernel: ROW, TMA tiles (16-byte aligned
// rows) or element-aligned tiles, with the kernel arguments.
enum QKind { kQRow = 0, kQTma = 1, kQTile = 2, kQShift = 3 };
struct QPlan {
  int kind, dtype, fmt, layout;
  bool aligned;  // ROW: chunks start 16-byte aligned in the input
  RowArgs ra;
  TileArgs ta;
  int off_e;     // kQShift: element offset of the input base inside its 16-byte granule
  CUtensorMap map;
};

int quantize_plan(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt, const RingArgs& r,
                  uint8_t* out, uint8_t* out_t, QPlan& q) {
  const int64_t n = rows * cols;
  const int eb = dtype == FP8_IN_FP32 ? 4 : 2;
  q = QPlan{};
  q.dtype = dtype;
  q.fmt = fmt;
  q.layout = layout;
  if (layout == FP8_LAYOUT_ROW) {
    RowArgs& a = q.ra;
    a.in = static_cast<const uint8_t*>(in);
    a.out = out;
    a.n = n;
    const uintptr_t oa = reinterpret_cast<uintptr_t>(out);
    a.head = std::min<int64_t>(n, int64_t((16 - (oa & 15)) & 15));
    a.nchunks = (n - a.head) / 16;
    a.ring = r;
    q.aligned = ((reinterpret_cast<uintptr_t>(in) + uintptr_t(a.head * eb)) & 15) == 0;
    q.kind = kQRow;
    return FP8_OK;
  }
  TileArgs& a = q.ta;
  a.in = static_cast<const uint8_t*>(in);
  a.out = out;
  a.out_t = out_t;
  a.rows = rows;
  a.cols = cols;
  a.tiles_c = (cols + kTileC - 1) / kTileC;
  a.ntiles = ((rows + kTileR - 1) / kTileR) * a.tiles_c;
  a.out8 = (layout == FP8_LAYOUT_DUAL) && (reinterpret_cast<uintptr_t>(out) % 8 == 0) && (cols % 8 == 0);
  a.outt4 = (reinterpret_cast<uintptr_t>(out_t) % 4 == 0) && (rows % 4 == 0);
  a.ring = r;
  if (n > 0 && reinterpret_cast<uintptr_t>(in) % 16 == 0 && (cols * eb) % 16 == 0 && a.ntiles < (int64_t(1) << 30) &&
      rows < (int64_t(1) << 30) && cols < (int64_t(1) << 30)) {
    if (!make_input_map(&q.map, in, dtype, rows, cols)) return FP8_ERR_CUDA;
    q.kind = kQTma;
  } else if (n > 0 && (cols * eb) % 16 == 0 && a.ntiles < (int64_t(1) << 30) && rows < (int64_t(1) << 30) &&
             cols < (int64_t(1) << 30)) {
    q.off_e = int((reinterpret_cast<uintptr_t>(in) & 15) / uintptr_t(eb));
    if (!make_shifted_map(&q.map, in, dtype, rows, cols, q.off_e)) return FP8_ERR_CUDA;
    q.kind = kQShift;
  } else {
    q.kind = kQTile;
  }
  return FP8_OK;
}

int quantize_launch(const QPlan& q, int sms, cudaStream_t st) {
  const bool dual = q.layout == FP8_LAYOUT_DUAL;
  if (q.kind == kQRow) {
    switch (q.dtype) {
      case FP8_IN_BF16: return dispatch_fmt_row<FP8_IN_BF16>(q.fmt, q.ra, sms, st, q.aligned);
      case FP8_IN_FP16: return dispatch_fmt_row<FP8_IN_FP16>(q.fmt, q.ra, sms, st, q.aligned);
      default: return dispatch_fmt_row<FP8_IN_FP32>(q.fmt, q.ra, sms, st, q.aligned);
    }
  }
  if (q.kind == kQTma || q.kind == kQShift) {
    const int off_e = q.kind == kQShift ? q.off_e : -1;
    switch (q.dtype) {
      case FP8_IN_BF16: return dispatch_fmt_tile_tma<FP8_IN_BF16>(q.fmt, q.ta, q.map, off_e, sms, st, dual);
      case FP8_IN_FP16: return dispatch_fmt_tile_tma<FP8_IN_FP16>(q.fmt, q.ta, q.map, off_e, sms, st, dual);
      default: return dispatch_fmt_tile_tma<FP8_IN_FP32>(q.fmt, q.ta, q.map, off_e, sms, st, dual);
    }
  }
  switch (q.dtype) {
    case FP8_IN_BF16: return dispatch_fmt_tile<FP8_IN_BF16>(q.fmt, q.ta, sms, st, dual);
    case FP8_IN_FP16: return dispatch_fmt_tile<FP8_IN_FP16>(q.fmt, q.ta, sms, st, dual);
    default: return dispatch_fmt_tile<FP8_IN_FP32>(q.fmt, q.ta, sms, st, dual);
  }
}

// Launches the cast kernel for the layout (and the ring fold unless r.history
// is null).  Arguments are already validated.
int quantize_dispatch(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt, const RingArgs& r,
                      uint8_t* out, uint8_t* out_t, cudaStream_t st) {
  const int sms = sm_count_current();
  if (sms <= 0) return FP8_ERR_CUDA;
  QPlan q;
  const int rc = quantize_plan(in, dtype, rows, cols, layout, fmt, r, out, out_t, q);
  return rc != FP8_OK ? rc : quantize_launch(q, sms, st);
}

// ---- several tensors in one launch -------------------------------------------

// One launch for n ROW plans with the same dtype and input alignment, each
// non-empty and on its own ring: the wave is shared in proportion to the
// chunks, and each tensor is sized as a single launch with its share (every
// thread the same number of chunks, at least kRowMinChunks).
template <int DT, bool kAligned>
int launch_row_multi1(const QPlan* const* qs, int n, int sms, cudaStream_t st) {
  static int cached[64] = {0};
  const int bps = resident_blocks(quantize_row_multi_kernel<DT, kAligned>, kRowThreads, cached);
  if (bps <= 0) return FP8_ERR_CUDA;
  const int64_t G = int64_t(bps) * sms;
  int64_t W = 0;
  for (int i = 0; i < n; ++i) W += qs[i]->ra.nchunks + 1;
  RowMultiArgs m;
  std::memset(&m, 0, sizeof(m));
  m.n = n;
  m.split[0] = 0;
  for (int i = 0; i < n; ++i) {
    const RowArgs& a = qs[i]->ra;
    const int64_t gmax = std::max<int64_t>(1, (G - n) * (a.nchunks + 1) / W);
    const int64_t tmax = gmax * kRowThreads;
    const int64_t per = std::max<int64_t>(kRowMinChunks, (a.nchunks + tmax - 1) / tmax);
    const int64_t g = std::max<int64_t>(1, (a.nchunks + per * kRowThreads - 1) / (per * kRowThreads));
    m.split[i + 1] = m.split[i] + unsigned(g);
    m.a[i] = a;
    m.fmt[i] = qs[i]->fmt;
  }
  const cudaError_t e = launch_pdl(quantize_row_multi_kernel<DT, kAligned>, dim3(m.split[n]), kRowThreads, 0, st, 1, m);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

int launch_row_multi(const QPlan* const* qs, int n, int sms, cudaStream_t st) {
  const bool al = qs[0]->aligned;
  switch (qs[0]->dtype) {
    case FP8_IN_BF16:
      return al ? launch_row_multi1<FP8_IN_BF16, true>(qs, n, sms, st)
                : launch_row_multi1<FP8_IN_BF16, false>(qs, n, sms, st);
    case FP8_IN_FP16:
      return al ? launch_row_multi1<FP8_IN_FP16, true>(qs, n, sms, st)
                : launch_row_multi1<FP8_IN_FP16, false>(qs, n, sms, st);
    default:
      return al ? launch_row_multi1<FP8_IN_FP32, true>(qs, n, sms, st)
                : launch_row_multi1<FP8_IN_FP32, false>(qs, n, sms, st);
  }
}

// ROW plans that can share one launch: same dtype and input alignment, each
// non-empty (formats may differ).
bool row_fusable(const QPlan* const* qs, int n) {
  for (int i = 0; i < n; ++i) {
    if (qs[i]->kind != kQRow || qs[i]->ra.n <= 0) return false;
    if (qs[i]->dtype != qs[0]->dtype || qs[i]->aligned != qs[0]->aligned) return false;
  }
  return true;
}

// One launch for n TMA-tile quantize plans with the same dtype and layout,
// each non-empty and each on its own ring: the wave of resident blocks is
// split between the tensors in proportion to their tiles (at least one block
// each, never more blocks than tiles).
template <int DT, bool kDual>
int launch_tile_tma_multi1(const QPlan* const* qs, int n, int sms, cudaStream_t st) {
  static int cached[64] = {0};
  auto kern = quantize_tile_tma_multi_kernel<DT, kDual>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FP8_ERR_CUDA;
  if (cached[dev] == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TmaTile<DT>::kSmem) != cudaSuccess)
      return FP8_ERR_CUDA;
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, kWsThreads, TmaTile<DT>::kSmem) != cudaSuccess || b < 1)
      return FP8_ERR_CUDA;
    cached[dev] = b;
  }
  const int64_t G = int64_t(cached[dev]) * sms;
  int64_t T = 0;
  for (int i = 0; i < n; ++i) T += qs[i]->ta.ntiles;
  const WaitCfg wc = wait_cfg();
  TmaMultiArgs m;
  std::memset(&m, 0, sizeof(m));
  m.n = n;
  m.split[0] = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t t = qs[i]->ta.ntiles;
    const int64_t g = std::min<int64_t>(t, std::max<int64_t>(1, (G - n) * t / T));
    m.split[i + 1] = m.split[i] + unsigned(g);
    m.maps[i] = qs[i]->map;
    m.a[i] = TmaTileArgs{qs[i]->ta, error_word_ptr(), wc.budget_ns, wc.stall_site, 0};
    m.fmt[i] = qs[i]->fmt;
  }
  const cudaError_t e = launch_pdl(kern, dim3(m.split[n]), kWsThreads, TmaTile<DT>::kSmem, st, 1, m);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

int launch_tile_tma_multi(const QPlan* const* qs, int n, int sms, cudaStream_t st) {
  const bool dual = qs[0]->layout == FP8_LAYOUT_DUAL;
  switch (qs[0]->dtype) {
    case FP8_IN_BF16:
      return dual ? launch_tile_tma_multi1<FP8_IN_BF16, true>(qs, n, sms, st)
                  : launch_tile_tma_multi1<FP8_IN_BF16, false>(qs, n, sms, st);
    case FP8_IN_FP16:
      return dual ? launch_tile_tma_multi1<FP8_IN_FP16, true>(qs, n, sms, st)
                  : launch_tile_tma_multi1<FP8_IN_FP16, false>(qs, n, sms, st);
    default:
      return dual ? launch_tile_tma_multi1<FP8_IN_FP32, true>(qs, n, sms, st)
                  : launch_tile_tma_multi1<FP8_IN_FP32, false>(qs, n, sms, st);
  }
}

// TMA-tile plans that can share one launch: same dtype and layout, each
// non-empty (formats may differ).
bool tma_fusable(const QPlan* const* qs, int n) {
  for (int i = 0; i < n; ++i) {
    if (qs[i]->kind != kQTma || qs[i]->ta.ntiles <= 0) return false;
    if (qs[i]->dtype != qs[0]->dtype || qs[i]->layout != qs[0]->layout) return false;
  }
  return true;
}

// Calls (on distinct rings) in one launch when they resolve to the same
// kernel -- ROW with the same dtype and alignment, or TMA tiles with the same
// dtype and layout -- and none is empty; otherwise one launch each, in order.
int quantize_multi_dispatch(const QPlan* const* qs, int n, cudaStream_t st) {
  const int sms = sm_count_current();
  if (sms <= 0) return FP8_ERR_CUDA;
  if (n > 1 && tma_fusable(qs, n)) return launch_tile_tma_multi(qs, n, sms, st);
  if (n > 1 && row_fusable(qs, n)) return launch_row_multi(qs, n, sms, st);
  for (int i = 0; i < n; ++i) {
    const int rc = quantize_launch(*qs[i], sms, st);
    if (rc != FP8_OK) return rc;
  }
  return FP8_OK;
}

}  // namespace
}  // namespace fp8ds

// Argument checks shared by the quantize entry points; FP8_OK if the call may
// proceed.
static int check_quantize_args(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt,
                               uint8_t* out, uint8_t* out_t, const uint32_t* scratch) {
  if (dtype < FP8_IN_BF16 || dtype > FP8_IN_FP32) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  if (layout < FP8_LAYOUT_ROW || layout > FP8_LAYOUT_DUAL) return FP8_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return FP8_ERR_INVALID_ARG;
  if (cols > 0 && rows > INT64_MAX / cols) return FP8_ERR_INVALID_ARG;
  if (scratch == nullptr) return FP8_ERR_INVALID_ARG;
  const int64_t n = rows * cols;
  if (n > 0 && in == nullptr) return FP8_ERR_INVALID_ARG;
  if ((layout == FP8_LAYOUT_ROW || layout == FP8_LAYOUT_DUAL) && n > 0 && out == nullptr) return FP8_ERR_INVALID_ARG;
  if ((layout == FP8_LAYOUT_T || layout == FP8_LAYOUT_DUAL) && n > 0 && out_t == nullptr) return FP8_ERR_INVALID_ARG;
  const int eb = dtype == FP8_IN_FP32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(in) % eb != 0) return FP8_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(scratch) % 8 != 0) return FP8_ERR_UNSUPPORTED;
  return FP8_OK;
}

extern "C" int fp8_quantize(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt,
                            fp8_ring ring, uint8_t* out, uint8_t* out_t, fp8_stream_t stream) {
  if (!ring.history || !ring.idx || !ring.scale || !ring.scale_inv || !ring.scratch) return FP8_ERR_INVALID_ARG;
  const int rc = check_quantize_args(in, dtype, rows, cols, layout, fmt, out, out_t, ring.scratch);
  if (rc != FP8_OK) return rc;
  const RingArgs r{ring.history, ring.idx, ring.scale, ring.scale_inv, ring.scratch};
  return quantize_dispatch(in, dtype, rows, cols, layout, fmt, r, out, out_t, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int fp8_quantize_pair(const fp8_quantize_args* q0, const fp8_quantize_args* q1, fp8_stream_t stream) {
  if (q0 == nullptr || q1 == nullptr) return FP8_ERR_INVALID_ARG;
  QPlan p[2];
  const fp8_quantize_args* qs[2] = {q0, q1};
  for (int i = 0; i < 2; ++i) {
    const fp8_quantize_args& q = *qs[i];
    const fp8_ring& ring = q.ring;
    if (!ring.history || !ring.idx || !ring.scale || !ring.scale_inv || !ring.scratch) return FP8_ERR_INVALID_ARG;
    const int rc = check_quantize_args(q.in, q.dtype, q.rows, q.cols, q.layout, q.fmt, q.out, q.out_t, ring.scratch);
    if (rc != FP8_OK) return rc;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int i = 0; i < 2; ++i) {
    const fp8_quantize_args& q = *qs[i];
    const RingArgs r{q.ring.history, q.ring.idx, q.ring.scale, q.ring.scale_inv, q.ring.scratch};
    const int rc = quantize_plan(q.in, q.dtype, q.rows, q.cols, q.layout, q.fmt, r, q.out, q.out_t, p[i]);
    if (rc != FP8_OK) return rc;
  }
  // One ring for both: two calls in order, as the caller wrote them.
  const bool shared = q0->ring.scratch == q1->ring.scratch || q0->ring.history == q1->ring.history;
  const QPlan* ptrs[2] = {&p[0], &p[1]};
  if (!shared) return quantize_multi_dispatch(ptrs, 2, st);
  const int rc = quantize_multi_dispatch(ptrs, 1, st);
  return rc != FP8_OK ? rc : quantize_multi_dispatch(ptrs + 1, 1, st);
}

extern "C" int fp8_quantize_multi(const fp8_quantize_args* qs, int n, fp8_stream_t stream) {
  if (qs == nullptr || n < 1 || n > kMaxMulti) return FP8_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const fp8_ring& ring = qs[i].ring;
    if (!ring.history || !ring.idx || !ring.scale || !ring.scale_inv || !ring.scratch) return FP8_ERR_INVALID_ARG;
    const int rc = check_quantize_args(qs[i].in, qs[i].dtype, qs[i].rows, qs[i].cols, qs[i].layout, qs[i].fmt,
                                       qs[i].out, qs[i].out_t, ring.scratch);
    if (rc != FP8_OK) return rc;
  }
  QPlan p[kMaxMulti];
  const QPlan* ptrs[kMaxMulti];
  for (int i = 0; i < n; ++i) {
    const fp8_ring& ring = qs[i].ring;
    const RingArgs r{ring.history, ring.idx, ring.scale, ring.scale_inv, ring.scratch};
    const int rc = quantize_plan(qs[i].in, qs[i].dtype, qs[i].rows, qs[i].cols, qs[i].layout, qs[i].fmt, r,
                                 qs[i].out, qs[i].out_t, p[i]);
    if (rc != FP8_OK) return rc;
    ptrs[i] = &p[i];
  }
  bool distinct = true;  // a ring cannot serve two calls of one launch
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j)
      if (qs[i].ring.scratch == qs[j].ring.scratch || qs[i].ring.history == qs[j].ring.history) distinct = false;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (distinct) return quantize_multi_dispatch(ptrs, n, st);
  for (int i = 0; i < n; ++i) {
    const int rc = quantize_multi_dispatch(ptrs + i, 1, st);
    if (rc != FP8_OK) return rc;
  }
  return FP8_OK;
}

extern "C" int fp8_quantize_local(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt,
                                  fp8_ring ring, float* amax_out, uint8_t* out, uint8_t* out_t,
                                  fp8_stream_t stream) {
  if (!ring.scale || !ring.scale_inv || !ring.scratch || !amax_out) return FP8_ERR_INVALID_ARG;
  const int rc = check_quantize_args(in, dtype, rows, cols, layout, fmt, out, out_t, ring.scratch);
  if (rc != FP8_OK) return rc;
  const RingArgs r{ring.history, ring.idx, ring.scale, ring.scale_inv, ring.scratch, amax_out};
  return quantize_dispatch(in, dtype, rows, cols, layout, fmt, r, out, out_t, reinterpret_cast<cudaStream_t>(stream));
}

namespace fp8ds {
namespace {
// The ring fold alone, of a given amax: one thread.  Same arithmetic as the
// last block of a quantize call (history write, max over the window, scale =
// FP8_MAX / max when positive, finite and finite in quotient; scale_inv =
// 1 / the scale in effect before the fold).
template <int FMT>
__global__ void ring_fold_kernel(float* history, int32_t* idx_p, float* scale, float* scale_inv, const float* amax) {
  pdl_launch_dependents();
  pdl_wait_prior_grid();
  if (threadIdx.x != 0) return;
  float hist[kHistoryLen];
#pragma unroll
  for (int i = 0; i < kHistoryLen; ++i) hist[i] = history[i];
  ring_commit<FMT>(*amax, hist, *idx_p, history, idx_p, scale, scale_inv, *scale);
}
}  // namespace
}  // namespace fp8ds

extern "C" int fp8_ring_fold(fp8_ring ring, int fmt, const float* amax, fp8_stream_t stream) {
  if (!ring.history || !ring.idx || !ring.scale || !ring.scale_inv || !amax) return FP8_ERR_INVALID_ARG;
  if (fmt != FP8_E4M3 && fmt != FP8_E5M2) return FP8_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e =
      fmt == FP8_E4M3
          ? launch_pdl(ring_fold_kernel<FP8_E4M3>, dim3(1), dim3(32), 0, st, 1, ring.history, ring.idx, ring.scale,
                       ring.scale_inv, amax)
          : launch_pdl(ring_fold_kernel<FP8_E5M2>, dim3(1), dim3(32), 0, st, 1, ring.history, ring.idx, ring.scale,
                       ring.scale_inv, amax);
  return e == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

extern "C" int fp8_quantize_current(const void* in, int dtype, int64_t rows, int64_t cols, int layout, int fmt,
                                    float* scale, float* scale_inv, float* amax, uint32_t* scratch, uint8_t* out,
                                    uint8_t* out_t, fp8_stream_t stream) {
  if (scale == nullptr || scale_inv == nullptr) return FP8_ERR_INVALID_ARG;
  const int rc = check_quantize_args(in, dtype, rows, cols, layout, fmt, out, out_t, scratch);
  if (rc != FP8_OK) return rc;
  const int sms = sm_count_current();
  if (sms <= 0) return FP8_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = rows * cols;
  const int eb = dtype == FP8_IN_FP32 ? 4 : 2;
  AmaxArgs a{};
  a.in = static_cast<const uint8_t*>(in);
  a.n = n;
  const uintptr_t ia = reinterpret_cast<uintptr_t>(in);
  a.head = std::min<int64_t>(n, int64_t(((16 - (ia & 15)) & 15) / eb));
  a.nchunks = (n - a.head) / 16;
  a.scratch = scratch;
  a.scale = scale;
  a.scale_inv = scale_inv;
  a.amax_out = amax;
  const int64_t want = (a.nchunks + 2 * kThreads - 1) / (2 * kThreads);
  const int grid = int(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(sms) * (2048 / kThreads))));
  cudaError_t e;
  switch (dtype * 2 + fmt) {
    case 0: e = launch_pdl(amax_kernel<FP8_IN_BF16, FP8_E4M3>, grid, kThreads, 0, st, 1, a); break;
    case 1: e = launch_pdl(amax_kernel<FP8_IN_BF16, FP8_E5M2>, grid, kThreads, 0, st, 1, a); break;
    case 2: e = launch_pdl(amax_kernel<FP8_IN_FP16, FP8_E4M3>, grid, kThreads, 0, st, 1, a); break;
    case 3: e = launch_pdl(amax_kernel<FP8_IN_FP16, FP8_E5M2>, grid, kThreads, 0, st, 1, a); break;
    case 4: e = launch_pdl(amax_kernel<FP8_IN_FP32, FP8_E4M3>, grid, kThreads, 0, st, 1, a); break;
    default: e = launch_pdl(amax_kernel<FP8_IN_FP32, FP8_E5M2>, grid, kThreads, 0, st, 1, a); break;
  }
  if (e != cudaSuccess) return FP8_ERR_CUDA;
  const RingArgs r{nullptr, nullptr, scale, scale_inv, scratch};
  return quantize_dispatch(in, dtype, rows, cols, layout, fmt, r, out, out_t, st);
}

// ---- variant for callers that cannot allocate --------------------------------
//
// Some callers cannot allocate device memory when they call us: operator or
// plugin interfaces that hand over only input and output pointers, and
// deployments that reserve all device memory at start-up (a cudaMalloc at run
// time can also synchronise the device and stall other streams).  For them
// fp8_quantize_static_scratch keeps the four scratch words that fp8_quantize
// takes from ring.scratch (amax bits, block ticket, tile counter, spare) in
// the library-owned array below instead.  Each GPU that loads the library
// holds these 256 bytes until the process exits.  All calls on a device share
// the array, so calls that overlap on the GPU race with each other.

#include <mutex>

static __device__ __align__(256) uint32_t g_quantize_static_scratch[64];

namespace {
constexpr int kStaticScratchWords = 64;    // capacity of g_quantize_static_scratch
constexpr int kQuantizeScratchWords = 4;   // what one quantize call needs, whatever its size

std::mutex g_static_scratch_mu;
uint32_t* g_static_scratch_ptr[64] = {nullptr};

// Device address of the static array on the current device, looked up once per
// device with that device current.  Host code must not use the symbol itself:
// on the host it is only a stand-in, not a device address.  A device reset
// (cudaDeviceReset) unloads the module and makes the cached address stale;
// the header says that this entry point must not be used after one.
uint32_t* static_scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (g_static_scratch_ptr[dev] == nullptr) {
    uint32_t* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_quantize_static_scratch) != cudaSuccess) return nullptr;
    g_static_scratch_ptr[dev] = p;
  }
  return g_static_scratch_ptr[dev];
}
}  // namespace

extern "C" int fp8_quantize_static_scratch(const void* in, int dtype, int64_t rows, int64_t cols, int layout,
                                           int fmt, fp8_ring ring, uint8_t* out, uint8_t* out_t,
                                           fp8_stream_t stream) {
  if (kQuantizeScratchWords > kStaticScratchWords) return FP8_ERR_UNSUPPORTED;
  if (!ring.history || !ring.idx || !ring.scale || !ring.scale_inv) return FP8_ERR_INVALID_ARG;
  uint32_t* scratch = static_scratch_on_current_device();
  if (scratch == nullptr) return FP8_ERR_CUDA;
  // Every argument check of fp8_quantize runs before the memset, so a
  // rejected call enqueues nothing.
  const int rc = check_quantize_args(in, dtype, rows, cols, layout, fmt, out, out_t, scratch);
  if (rc != FP8_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The kernel leaves the words at zero when it finishes; clearing them here
  // as well means a call never depends on what an earlier call left behind.
  if (cudaMemsetAsync(scratch, 0, kQuantizeScratchWords * sizeof(uint32_t), st) != cudaSuccess) return FP8_ERR_CUDA;
  const RingArgs r{ring.history, ring.idx, ring.scale, ring.scale_inv, scratch};
  return quantize_dispatch(in, dtype, rows, cols, layout, fmt, r, out, out_t, st);
}
