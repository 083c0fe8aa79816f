// sq_linear_tc.cu -- the decode linear layer on the tensor cores (sm_100a),
// for weights packed in SQ_LAYOUT_TILES.
//
// Page: "1-bit量化不是玄学，以往掉点是机制问题" (m.lqnn.cn/news/241359),
// section 2.3: the 1-bit trunk product and the high-bit residual product are
// computed side by side and summed; section 3.3: all of it in one kernel.
//
// Same results as sq_linear.cu (bit-exact integer accumulators, fp32 y), up
// to 8 tokens per pass (the MMA's N):
//   * residual: four int8 MMAs (mma.sync m16n8k32) per tile of 16 rows x 128
//     channels give the exact group sums R_g; each lane's 64 bytes of the
//     tile are already its four A fragments (the packed layout is the MMA's
//     operand order), so they go from the warp's shared-memory ring straight
//     into the MMAs;
//   * trunk: the sign bits are stored so that the four bits of one 4-channel
//     word are the top bits of the four bytes of (bits << (7 - w)); a
//     sign-replicating byte permute (prmt) turns them into 0 / -1 bytes, one
//     shift and one permute per word, and the same int8 MMAs against the same
//     activation codes give -P = -sum_{m and b} xq; S = sum_m xq comes from an
//     all-ones (or the mask's) operand; T = 2P - S.  (A binary AND/popcount
//     MMA would read the bits directly, but sm_100 runs it emulated at ~69
//     instructions per m16n8k128, ten times the int8 MMA.)
// Work: one CTA of 16 warps per SM owns whole row blocks; its tiles, in
// row-block-major order, are split evenly over its warps.  The packed tiles
// lie in memory in that same order, so each warp streams one contiguous range
// (through a per-warp cp.async ring in shared memory) with no edge cases: rows
// and channels are zero padded.  A row block finished inside one warp is
// written at once; one shared by warps of the CTA is summed from shared memory
// after one CTA barrier, in warp order, so the results do not depend on timing.
// Fused mode (sq_quantize_linear): the kernel takes the fp32 activations and
// performs the activation split itself after the weight prefetch: every CTA
// forms the per-token scale (absmax over the non-outlier channels), the INT8
// codes and the outlier values in shared memory with the same arithmetic as
// the activation split kernel, and the main loop reads its codes from there.
#include <stdint.h>

#include <algorithm>
#include <cstdint>

#include "sq_common.cuh"
#include "sq_internal.h"
#include "sq_layout.h"
#include "sq_quant.cuh"

namespace sq {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kBps = 1;    // CTAs per SM
// Fused mode: tiles copied before the activation split.  The split's loads
// of x must not queue behind a full ring of weight loads, so only the first
// tile is in flight while it runs; the rest follow it.
constexpr int kDepthEarly = 1;
// Tiles in flight per warp (the shared-memory ring).  Deeper rings measured
// slower: two tiles per warp keep enough bytes in flight at batch <= 2, three
// above it, where a tile takes longer to consume.
constexpr int kDeep = 3, kShallow = 2;
constexpr int kCols = 8;   // tokens per pass (MMA N)

struct Params {
  const int8_t* res;
  const uint32_t* sign;
  const uint32_t* mask;
  const float* alpha;
  const float* scale;
  const uint32_t* keep;    // keep bits of a sparse residual (SQ_LAYOUT_TILES_SPARSE)
  const int32_t* nbytes;   // packed code bytes per tile (sparse)
  const int32_t* zero;     // zero-points of an asymmetric residual (SQ_LAYOUT_TILES_ASYM)
  int N, K, tpr;    // rows, channels, tiles per row block
  int T;            // tiles = ceil(N / 16) * tpr
  int n_rb;         // row blocks = ceil(N / 16); CTA b owns [b*n_rb/grid, (b+1)*n_rb/grid)
  int M;            // tokens in this pass (<= 8)
  const int8_t* xq;
  int xs;           // row stride of xq (roundup(K, 128))
  const float* sx;
  const float* xout;
  const int32_t* idx;
  int n_out;
  float* y;
  int32_t* T_out;
  int32_t* R_out;
  int pdl;
  // fused mode
  const float* x;     // [M][K] activations
  int32_t* status;    // device status word (non-finite x, bad index list)
  int n_pad;          // x_out row stride in shared memory
  int off_xq, off_xo, off_sx, off_red;  // shared-memory offsets (bytes)
  // shared-memory offsets of the tile rings and the outlier bitmap (bytes)
  int off_ring, off_omask;
};

// Work split: CTA b owns whole row blocks [b*n_rb/grid, (b+1)*n_rb/grid), so
// no row block is shared between CTAs; its tiles are split evenly over its
// warps (a row block may be shared by warps of the CTA).
__device__ __forceinline__ int cta_first_tile(int b, const Params& p) {
  return (int)((int64_t)b * p.n_rb / gridDim.x) * p.tpr;
}
// First tile of warp i of the CTA whose tiles are [T0, T1).
__device__ __forceinline__ int warp_first_tile(int i, int T0, int T1) {
  return T0 + (int)((int64_t)i * (T1 - T0) / kWarps);
}
// The warp of that CTA whose range holds tile t.
__device__ __forceinline__ int tile_warp(int t, int T0, int T1) {
  const int len = T1 - T0;
  return (int)(((int64_t)(t - T0 + 1) * kWarps + len - 1) / len) - 1;
}

__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte k of the result = 0xFF if bit 8k+7 of x is set, else 0 (prmt with
// the sign-replicate bit in every selector nibble).
__device__ __forceinline__ uint32_t sign_bytes(uint32_t x) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, 0xBA98;" : "=r"(d) : "r"(x));
  return d;
}
// Channels 4w .. 4w+3 of a lane's 32 as 0 / -1 bytes (tiled bit order).
__device__ __forceinline__ uint32_t bits_word(uint32_t bits, int w) {
  return sign_bytes(bits << (7 - w));
}

// One tile as seen by one lane.
template <bool MASK>
struct Tile {
  uint32_t q[16];  // four A fragments of residual codes
  uint32_t s[2];   // sign words of rows r0, r1
  uint32_t m[2];   // mask words (MASK only)
  float c[2];      // group scales of rows r0, r1
  int z[2];        // zero-points of rows r0, r1 (asymmetric residual only)
};

// Streaming position of one lane: its part of the next tile to copy.
struct Cursor {
  const uint8_t* code;   // the tile's code bytes + 16 * lane; + 2048 per tile
  const uint32_t* sign;  // the lane's two sign words; + 64 words per tile
  const uint32_t* mask;
  const float* scale;    // the scale of row r0 (r1: + 8); + 16 floats per tile
  // sparse residual: the lane's two keep words, and the packed code bytes of
  // the cursor's tile (loaded one tile ahead, 0 past the last tile)
  const uint32_t* keep;
  const int32_t* nbytes;
  int nb, t, T;
  const int32_t* zero;   // asymmetric residual: the zero-point of row r0 (r1: + 8)
  template <bool SPARSE, bool ASYM = false>
  __device__ __forceinline__ void advance() {
    code += 2048;
    sign += 64;
    mask += 64;
    scale += 16;
    if constexpr (ASYM) zero += 16;
    if constexpr (SPARSE) {
      keep += 64;
      ++nbytes;
      ++t;
      nb = t < T ? __ldg(nbytes) : 0;
    }
  }
};

// ---- shared-memory tile ring ------------------------------------------------------
// Each warp streams its tiles through a ring of D slots filled by cp.async
// (global -> shared without registers), D tiles ahead of use.  Slot layout:
// 32 lanes x 64 code bytes, then 32 x 8 sign bytes (then 32 x 8 mask bytes),
// then 32 x 8 bytes of the lane's two scales.  Code chunk j (16 bytes) of lane
// L sits at L*64 + ((j + L/2) % 4) * 16, so the 16-byte reads of eight
// consecutive lanes hit eight different bank groups.
// The codes are copied in four warp-wide instructions of 512 contiguous bytes
// (whole 32-byte sectors, each requested once), 16 bytes per lane, into their
// owners' places, so the warp synchronises after the wait (the owner reads
// other lanes' copies) and before a refill (no lane may still read the slot).
// They bypass L1.  A lane copies its own sign, mask and scale words, through
// L1, where neighbouring lanes' requests coalesce (16-byte copies that bypass
// L1 measured slower for these).
// In the trunk-only mode (RES = false) a slot holds only the 256 sign bytes
// (then the 256 mask bytes), and the ring is kTrunkDepth slots deep.
// A sparse residual (SPARSE) keeps the tile's packed codes, as they lie in
// memory, in the code area and its keep words after the bit planes.
// An asymmetric residual (ASYM) keeps the lane's two zero-points after the scales.
template <bool MASK, bool RES = true, bool SPARSE = false, bool ASYM = false>
struct Slot {
  static constexpr int kSign = RES ? 2048 : 0;
  static constexpr int kMask = kSign + 256;  // (MASK only)
  static constexpr int kKeep = MASK ? kMask + 256 : kMask;  // (SPARSE only)
  static constexpr int kScale = SPARSE ? kKeep + 256 : kKeep;  // (RES only)
  static constexpr int kZero = kScale + 256;  // (ASYM only)
  static constexpr int kBytes = ASYM ? kZero + 256 : kScale + (RES ? 256 : 0);
};
// Tiles in flight per warp in the trunk-only mode (small slots).
constexpr int kTrunkDepth = 6;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// All but the newest N groups of this thread's copies are complete.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// RES = false (trunk only): the codes and scales are neither copied nor read.
// SPARSE: only the tile's c.nb packed code bytes are copied, as they lie.
template <bool MASK, bool RES, bool SPARSE = false, bool ASYM = false>
__device__ __forceinline__ void copy_tile(uint32_t slot, const Cursor& c, int lane) {
  using SL = Slot<MASK, RES, SPARSE, ASYM>;
  if constexpr (RES && SPARSE) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if ((lane + 32 * j) * 16 < c.nb) cp_async16(slot + lane * 16 + 512 * j, c.code + 512 * j);
    cp_async8(slot + SL::kKeep + lane * 8, c.keep);
  } else if constexpr (RES) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int lo = j * 8 + (lane >> 2), ch = lane & 3;  // owner lane, its chunk
      cp_async16(slot + lo * 64 + (((ch + (lo >> 1)) & 3) << 4), c.code + 512 * j);
    }
  }
  cp_async8(slot + SL::kSign + lane * 8, c.sign);
  if constexpr (MASK) cp_async8(slot + SL::kMask + lane * 8, c.mask);
  if constexpr (RES) {
    cp_async4(slot + SL::kScale + lane * 8, c.scale);
    cp_async4(slot + SL::kScale + lane * 8 + 4, c.scale + 8);
  }
  if constexpr (ASYM) {
    cp_async4(slot + SL::kZero + lane * 8, c.zero);
    cp_async4(slot + SL::kZero + lane * 8 + 4, c.zero + 8);
  }
}

// Sparse residual: the lane's codes from the tile's packed stream.  Its
// place in the stream is the count of kept codes of the lanes before it (a
// warp scan of the keep-bit counts); each 4-channel word (row r0's 32
// channels, then row r1's) takes the next popc(keep nibble) bytes, spread to
// its kept channels by one byte permute whose selector comes from a 16-entry
// table (sel_lut[n]: byte c from stream byte popc(n & ((1 << c) - 1)) if bit
// c of n is set, else 0).  (Forming the 16 words independently, each from its
// own popcount offset, measured slower: the reads of shared memory, not their
// latency, bound this expansion.)
__device__ __forceinline__ void expand_sparse(uint32_t (&q)[16], const uint8_t* slot, uint32_t k0,
                                              uint32_t k1, int lane, const uint32_t* sel_lut) {
  const int n = __popc(k0) + __popc(k1);
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int pos = incl - n;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(slot);
  uint32_t lo = cw[pos >> 2], hi = cw[(pos >> 2) + 1];
#pragma unroll
  for (int R = 0; R < 2; ++R) {
    const uint32_t kb = R ? k1 : k0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      // keep bits 8c + w of the word are channels 4w + c
      const uint32_t nib = (((kb >> w) & 0x01010101u) * 0x01020408u) >> 24;
      const uint32_t bytes = __funnelshift_r(lo, hi, (pos & 3) * 8);
      q[4 * (w >> 1) + 2 * (w & 1) + R] = __byte_perm(bytes, 0u, sel_lut[nib]);
      const int np = pos + __popc(nib);
      if ((np >> 2) != (pos >> 2)) {
        lo = hi;
        hi = cw[(np >> 2) + 1];
      }
      pos = np;
    }
  }
}

template <bool MASK, bool RES, bool SPARSE = false, bool ASYM = false>
__device__ __forceinline__ void read_tile(Tile<MASK>& t, const uint8_t* slot, int lane,
                                          const uint32_t* sel_lut = nullptr) {
  using SL = Slot<MASK, RES, SPARSE, ASYM>;
  if constexpr (RES && SPARSE) {
    const uint2 kv = *reinterpret_cast<const uint2*>(slot + SL::kKeep + lane * 8);
    expand_sparse(t.q, slot, kv.x, kv.y, lane, sel_lut);
  } else if constexpr (RES) {
    const uint8_t* cb = slot + lane * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = *reinterpret_cast<const uint4*>(cb + (((j + (lane >> 1)) & 3) << 4));
      t.q[4 * j] = v.x;
      t.q[4 * j + 1] = v.y;
      t.q[4 * j + 2] = v.z;
      t.q[4 * j + 3] = v.w;
    }
  }
  const uint2 sv = *reinterpret_cast<const uint2*>(slot + SL::kSign + lane * 8);
  t.s[0] = sv.x;
  t.s[1] = sv.y;
  if constexpr (MASK) {
    const uint2 mv = *reinterpret_cast<const uint2*>(slot + SL::kMask + lane * 8);
    t.m[0] = mv.x;
    t.m[1] = mv.y;
  }
  if constexpr (RES) {
    const float2 cv = *reinterpret_cast<const float2*>(slot + SL::kScale + lane * 8);
    t.c[0] = cv.x;
    t.c[1] = cv.y;
  }
  if constexpr (ASYM) {
    const int2 zv = *reinterpret_cast<const int2*>(slot + SL::kZero + lane * 8);
    t.z[0] = zv.x;
    t.z[1] = zv.y;
  }
}

// Code of channel j (0..31) of row R (0: r0, 1: r1) held in a tile's A
// fragments: register 4*(w/2) + 2*(w%2) + R of word w = j/4 (static
// register indices only, selected by the bits of w).
template <int R>
__device__ __forceinline__ int tile_code(const uint32_t* q, int j) {
  const int w = j >> 2;
  const bool o = w & 1;
  const uint32_t x01 = o ? q[2 + R] : q[0 + R];
  const uint32_t x23 = o ? q[6 + R] : q[4 + R];
  const uint32_t x45 = o ? q[10 + R] : q[8 + R];
  const uint32_t x67 = o ? q[14 + R] : q[12 + R];
  const uint32_t lo = (w & 2) ? x23 : x01, hi = (w & 2) ? x67 : x45;
  const uint32_t v = (w & 4) ? hi : lo;
  return (int)(int8_t)(v >> (8 * (j & 3)));
}

// Per-lane sums of one row-block piece: rows (r0, r1) x tokens (tk0, tk1),
// in MMA accumulator order (r0 tk0, r0 tk1, r1 tk0, r1 tk1).
struct Acc {
  int Pn[4];     // -sum_{m and b} xq
  int S[4];      // sum xq (no mask) or -sum_m xq (mask)
  float F[4];    // sum_g s_g R_g
  float Ut[4];   // outlier trunk part: sum (+-1 or 0) * x_out
  float Ur[4];   // outlier residual part: sum s_g q * x_out
};

__device__ __forceinline__ void acc_zero(Acc& a) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a.Pn[i] = 0;
    a.S[i] = 0;
    a.F[i] = 0.0f;
    a.Ut[i] = 0.0f;
    a.Ur[i] = 0.0f;
  }
}

// T = 2P - S
template <bool MASK>
__device__ __forceinline__ int trunk_T(const Acc& a, int i) {
  return MASK ? -2 * a.Pn[i] + a.S[i] : -2 * a.Pn[i] - a.S[i];
}

__device__ __forceinline__ float4 cell(int T, float F, float Ut, float Ur) {
  return make_float4(__int_as_float(T), F, Ut, Ur);
}
__device__ __forceinline__ void cell_add(float4& a, const float4& b) {
  a.x = __int_as_float(__float_as_int(a.x) + __float_as_int(b.x));
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}

// y of this lane's four (row, token) cells of row block rb:
// y = sx * (alpha * T + F) + (alpha * Ut + Ur).
__device__ __forceinline__ void write_y(const Params& p, int rb, int gid, int tid4,
                                        const float4 (&v)[4], float al0, float al1, float sx0,
                                        float sx1, int tko) {
  const int r0 = rb * kTileRows + gid, r1 = r0 + 8;
  const int tk0 = 2 * tid4 + tko, tk1 = tk0 + 1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = (i < 2) ? r0 : r1, tk = (i & 1) ? tk1 : tk0;
    const float al = (i < 2) ? al0 : al1, s = (i & 1) ? sx1 : sx0;
    if (row < p.N && tk < p.M)
      p.y[(int64_t)tk * p.N + row] =
          fmaf(s, fmaf(al, (float)__float_as_int(v[i].x), v[i].y), fmaf(al, v[i].z, v[i].w));
  }
}

// Fused mode: the activation split of the pass's tokens into shared memory
// (codes [M][K128], outlier values [M][n_pad], scales [M]); outlier channels
// are those marked in omask.  Same arithmetic as the activation split kernel.
// Latency is what counts here (the weight stream waits for the codes): for
// K <= 16384 each thread keeps its share of a token's x in registers (float4,
// all loads in flight at once), so a token costs one memory round trip and
// one barrier; the outlier values are gathered with the same round trip.
// float4 per thread kept in registers: K <= 16384 (16 per thread made the
// compiler spill registers in the fused kernels)
constexpr int kXRegs = 8;

// jv, jp: this thread's entry of the outlier list and the one before it
// (threads < n_out, loaded in the prologue).
__device__ __forceinline__ void split_activations(const Params& p, const uint32_t* omask,
                                                  int8_t* xq_s, float* xo_s, float* sx_s,
                                                  float* red_s, int jv, int jp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K128 = p.xs;
  const int K4 = p.K >> 2, Kq = K128 >> 2;
  const bool vec = (p.K & 3) == 0 && (reinterpret_cast<uintptr_t>(p.x) & 15u) == 0;
  const bool in_regs = vec && Kq <= kXRegs * kThreads;
  bool nonfinite = false;
  bool bad_idx = false;
  // the index list is checked once (strictly ascending, inside [0, K))
  for (int i = threadIdx.x; i < p.n_out; i += kThreads) {
    const int j = i < kThreads ? jv : p.idx[i];
    const int jq = i < kThreads ? jp : p.idx[i - 1];
    bad_idx |= j < 0 || j >= p.K || (i > 0 && jq >= j);
  }
  for (int t = 0; t < p.M; ++t) {
    const float* xt = p.x + (int64_t)t * p.K;
    uint32_t* q4 = reinterpret_cast<uint32_t*>(xq_s + t * K128);
    // outlier values of this token, loaded alongside x
    if (threadIdx.x < p.n_out)
      xo_s[t * p.n_pad + threadIdx.x] = (jv >= 0 && jv < p.K) ? xt[jv] : 0.0f;
    for (int i = threadIdx.x + kThreads; i < p.n_out; i += kThreads) {
      const int j = p.idx[i];
      xo_s[t * p.n_pad + i] = (j >= 0 && j < p.K) ? xt[j] : 0.0f;
    }
    float a = 0.0f;
    float4 xr[kXRegs];
    if (in_regs) {
      const float4* x4 = reinterpret_cast<const float4*>(xt);
      // (every loop over u stops at a bound that is the same for the whole CTA)
#pragma unroll
      for (int u = 0; u < kXRegs; ++u) {
        if (u * kThreads >= K4) break;
        const int j4 = threadIdx.x + u * kThreads;
        xr[u] = j4 < K4 ? x4[j4] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
#pragma unroll
      for (int u = 0; u < kXRegs; ++u) {
        if (u * kThreads >= K4) break;
        const int j4 = threadIdx.x + u * kThreads;
        if (j4 < K4) a = absmax4(xr[u], omask_nibble(omask, j4), a, nonfinite);
      }
    } else if (vec) {
      const float4* x4 = reinterpret_cast<const float4*>(xt);
      for (int j4 = threadIdx.x; j4 < K4; j4 += kThreads) a = absmax4(x4[j4], omask_nibble(omask, j4), a, nonfinite);
    } else {
      for (int j = threadIdx.x; j < p.K; j += kThreads) {
        const float v = xt[j];
        nonfinite |= !isfinite(v);
        if (!((omask[j >> 5] >> (j & 31)) & 1u)) a = fmaxf(a, fabsf(v));
      }
    }
    // a >= 0 (or +inf): the order of non-negative floats is that of their bits
    a = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
    if (lane == 0) red_s[(t & 1) * kWarps + warp] = a;  // two buffers: token t+1 may start early
    __syncthreads();
    {
      const uint4* r4 = reinterpret_cast<const uint4*>(red_s + (t & 1) * kWarps);
      uint32_t m = 0u;
#pragma unroll
      for (int w = 0; w < kWarps / 4; ++w) {
        const uint4 v = r4[w];
        m = max(m, max(max(v.x, v.y), max(v.z, v.w)));
      }
      a = __uint_as_float(m);
    }
    const float s = act_scale(a);
    const float rinv = act_rinv(s);
    if (threadIdx.x == 0) sx_s[t] = s;
    // one branch per token: the common range needs no per-element test
    const bool fast = quantize_fast_ok(s, a);
    if (in_regs && fast) {
#pragma unroll
      for (int u = 0; u < kXRegs; ++u) {
        if (u * kThreads >= Kq) break;
        const int j4 = threadIdx.x + u * kThreads;
        if (j4 < Kq) q4[j4] = j4 < K4 ? pack_codes<true>(xr[u], omask_nibble(omask, j4), s, rinv) : 0u;
      }
    } else if (in_regs) {
#pragma unroll
      for (int u = 0; u < kXRegs; ++u) {
        if (u * kThreads >= Kq) break;
        const int j4 = threadIdx.x + u * kThreads;
        if (j4 < Kq) q4[j4] = j4 < K4 ? pack_codes<false>(xr[u], omask_nibble(omask, j4), s, rinv) : 0u;
      }
    } else if (vec) {
      const float4* x4 = reinterpret_cast<const float4*>(xt);
      for (int j4 = threadIdx.x; j4 < Kq; j4 += kThreads)
        q4[j4] = j4 < K4 ? pack_codes<false>(x4[j4], omask_nibble(omask, j4), s, rinv) : 0u;
    } else {
      for (int j = threadIdx.x; j < K128; j += kThreads) {
        int q = 0;
        if (j < p.K && !((omask[j >> 5] >> (j & 31)) & 1u)) q = quantize_exact(xt[j], s, rinv);
        xq_s[t * K128 + j] = (int8_t)q;
      }
    }
  }
  if (nonfinite) set_status(p.status, SQ_ERR_NONFINITE);
  if (bad_idx) set_status(p.status, SQ_ERR_INVALID_ARG);
  __syncthreads();
}

// RES = false: the trunk-only mode (the residual path skipped: no codes or
// scales read, no residual MMAs, outlier channels take the trunk weight).
// SPARSE: the weight is in SQ_LAYOUT_TILES_SPARSE (packed kept codes).
// ASYM: SQ_LAYOUT_TILES_ASYM: a group's residual term is s_g * (R_g - z_g * S_g)
// with S_g the sum of the group's activation codes, exact in 64-bit integers.
// NT: groups of 8 tokens per pass (the MMA's N); every tile's weights serve
// all of them, so a pass of 16 tokens reads the weights once.
template <bool MASK, bool EMIT, bool FUSED, int D, bool RES, bool SPARSE, bool ASYM, int NT>
__global__ void __launch_bounds__(kThreads, kBps) k_linear_tc(const Params p) {
  using SL = Slot<MASK, RES, SPARSE, ASYM>;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t sel_lut[16];  // byte-permute selectors of the sparse expansion
  // shared: part [kWarps][2 slots][16 rows][M tokens] float4 | omask[nw] u32 |
  // obase[nw] i32 | fused-mode buffers | ring [kWarps][D slots]
  float4* part_s = reinterpret_cast<float4*>(smem);
  const int nw = p.tpr * 4;  // 32-channel words of a padded row
  uint32_t* omask = reinterpret_cast<uint32_t*>(smem + p.off_omask);
  int* obase = reinterpret_cast<int*>(omask + nw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid4 = lane & 3;
  const int T0c = cta_first_tile(blockIdx.x, p), T1c = cta_first_tile(blockIdx.x + 1, p);
  const int t0 = warp_first_tile(warp, T0c, T1c), t1 = warp_first_tile(warp + 1, T0c, T1c);

  // ---- the outlier index list first (small loads ahead of the stream)
  const int my_i = threadIdx.x;
  const int jv = my_i < p.n_out ? __ldg(p.idx + my_i) : -1;
  const int jp = (my_i < p.n_out && my_i > 0) ? __ldg(p.idx + my_i - 1) : -1;
  for (int i = threadIdx.x; i < nw; i += kThreads) omask[i] = 0u;

  // ---- copy the first D tiles (weights only: allowed before the wait)
  Cursor cur;
  {
    const int64_t lt = (int64_t)t0 * 32 + lane;
    cur.code = reinterpret_cast<const uint8_t*>(p.res) + (int64_t)t0 * 2048 + lane * 16;
    cur.sign = p.sign + lt * 2;
    cur.mask = MASK ? p.mask + lt * 2 : p.sign;
    cur.scale = p.scale + (int64_t)t0 * 16 + gid;
    if constexpr (ASYM) cur.zero = p.zero + (int64_t)t0 * 16 + gid;
    if constexpr (SPARSE) {
      cur.keep = p.keep + lt * 2;
      cur.nbytes = p.nbytes + t0;
      cur.t = t0;
      cur.T = p.T;
      cur.nb = t0 < p.T ? __ldg(cur.nbytes) : 0;
    }
  }
  if (SPARSE && threadIdx.x < 16) {
    const uint32_t n = threadIdx.x;
    uint32_t sel = 0;
    for (int c = 0; c < 4; ++c)
      sel |= (((n >> c) & 1u) ? (uint32_t)__popc(n & ((1u << c) - 1u)) : 4u) << (4 * c);
    sel_lut[n] = sel;
  }
  uint8_t* ring_w = smem + p.off_ring + warp * D * SL::kBytes;
  const uint32_t ring_u = smem_u32(ring_w);
  constexpr int kEarly = FUSED ? kDepthEarly : D;
#pragma unroll
  for (int d = 0; d < kEarly; ++d) {  // one commit group per tile, empty past the range
    if (t0 + d < t1) copy_tile<MASK, RES, SPARSE, ASYM>(ring_u + d * SL::kBytes, cur, lane);
    cp_async_commit();
    cur.advance<SPARSE, ASYM>();
  }

  __syncthreads();  // omask zeroed (and the selector table written)
  auto add_outlier = [&](int i, int j, int jprev) {
    if (j >= 0 && j < p.K) {
      atomicOr(&omask[j >> 5], 1u << (j & 31));
      if (i == 0 || (jprev >> 5) != (j >> 5)) obase[j >> 5] = i;
    }
  };
  if (my_i < p.n_out) add_outlier(my_i, jv, jp);
  for (int i = my_i + kThreads; i < p.n_out; i += kThreads) add_outlier(i, p.idx[i], p.idx[i - 1]);
  if (FUSED && p.pdl) {
    // warm L2 with the activations while the previous kernel finishes (a
    // prefetch moves no data to the SM, so it cannot return stale values)
    const char* xb = reinterpret_cast<const char*>(p.x);
    const int64_t xbytes = (int64_t)p.M * p.K * 4;
    for (int64_t o = (int64_t)threadIdx.x * 128; o < xbytes; o += kThreads * 128)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(xb + o));
  }
  __syncthreads();
  if (p.pdl) {
    pdl_wait();
    pdl_launch_dependents();
  }
  int8_t* xq_s = reinterpret_cast<int8_t*>(smem + p.off_xq);
  float* xo_s = reinterpret_cast<float*>(smem + p.off_xo);
  float* sx_s = reinterpret_cast<float*>(smem + p.off_sx);
  if constexpr (FUSED) {
    split_activations(p, omask, xq_s, xo_s, sx_s, reinterpret_cast<float*>(smem + p.off_red), jv, jp);
#pragma unroll
    for (int d = kEarly; d < D; ++d) {
      if (t0 + d < t1) copy_tile<MASK, RES, SPARSE, ASYM>(ring_u + d * SL::kBytes, cur, lane);
      cp_async_commit();
      cur.advance<SPARSE, ASYM>();
    }
  }

  // tokens of this lane's accumulator columns in token group kg: tk0 + 8 kg
  // and tk1 + 8 kg; the B operand of this lane (MMA column gid) is token
  // min(gid + 8 kg, M - 1): columns past M are not written
  const int tk0 = 2 * tid4, tk1 = tk0 + 1;
  float sx0[NT], sx1[NT];
  const int8_t* xrow[NT];
  Acc acc[NT];
#pragma unroll
  for (int kg = 0; kg < NT; ++kg) {
    const int a0 = tk0 + 8 * kg, a1 = tk1 + 8 * kg;
    if constexpr (FUSED) {
      sx0[kg] = a0 < p.M ? sx_s[a0] : 0.0f;
      sx1[kg] = a1 < p.M ? sx_s[a1] : 0.0f;
    } else {
      sx0[kg] = a0 < p.M ? __ldg(p.sx + a0) : 0.0f;
      sx1[kg] = a1 < p.M ? __ldg(p.sx + a1) : 0.0f;
    }
    const int tok = min(gid + 8 * kg, p.M - 1);
    xrow[kg] = (FUSED ? xq_s + tok * p.xs : p.xq + (int64_t)tok * p.xs) + tid4 * 32;
    acc_zero(acc[kg]);
  }
  int rb = t0 / p.tpr, cg = t0 - rb * p.tpr;
  bool rb_head = (cg == 0);  // this piece starts at the row block's first tile
  float al0 = 0.0f, al1 = 0.0f;
  if (t0 < t1) {
    al0 = __ldg(p.alpha + rb * kTileRows + gid);
    al1 = __ldg(p.alpha + rb * kTileRows + gid + 8);
  }
  const uint32_t kOnes = 0x01010101u;

  int slot_i = 0;
  for (int t = t0; t < t1; ++t) {
    cp_async_wait<D - 1>();  // this lane's copies of the tile have landed
    __syncwarp();             // ... and every lane's
    Tile<MASK> tl;
    read_tile<MASK, RES, SPARSE, ASYM>(tl, ring_w + slot_i * SL::kBytes, lane, sel_lut);
    const uint32_t pb0 = MASK ? (tl.s[0] & tl.m[0]) : tl.s[0];
    const uint32_t pb1 = MASK ? (tl.s[1] & tl.m[1]) : tl.s[1];
#pragma unroll
    for (int kg = 0; kg < NT; ++kg) {
      Acc& ac = acc[kg];
      // activation codes of this lane's 32 channels for its MMA column
      uint32_t xw[8];
      {
        const int4* xp = reinterpret_cast<const int4*>(xrow[kg] + cg * kTileK);
        int4 a, b;
        if constexpr (FUSED) {
          a = xp[0];
          b = xp[1];
        } else {
          a = __ldg(xp);
          b = __ldg(xp + 1);
        }
        xw[0] = a.x; xw[1] = a.y; xw[2] = a.z; xw[3] = a.w;
        xw[4] = b.x; xw[5] = b.y; xw[6] = b.z; xw[7] = b.w;
      }
      int R[4] = {0, 0, 0, 0};
      // asymmetric residual: the tile's activation sum S_g per token, from the
      // all-ones MMA (the growth of ac.S over the tile; with a mask, its own)
      const int S0[4] = {ac.S[0], ac.S[1], ac.S[2], ac.S[3]};
      int Sg[4] = {0, 0, 0, 0};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t b0 = xw[2 * m], b1 = xw[2 * m + 1];
        if constexpr (RES)
          mma_s8(R, tl.q[4 * m], tl.q[4 * m + 1], tl.q[4 * m + 2], tl.q[4 * m + 3], b0, b1);
        mma_s8(ac.Pn, bits_word(pb0, 2 * m), bits_word(pb1, 2 * m), bits_word(pb0, 2 * m + 1),
               bits_word(pb1, 2 * m + 1), b0, b1);
        if constexpr (MASK)
          mma_s8(ac.S, bits_word(tl.m[0], 2 * m), bits_word(tl.m[1], 2 * m),
                 bits_word(tl.m[0], 2 * m + 1), bits_word(tl.m[1], 2 * m + 1), b0, b1);
        else
          mma_s8(ac.S, kOnes, kOnes, kOnes, kOnes, b0, b1);
        if constexpr (ASYM && MASK) mma_s8(Sg, kOnes, kOnes, kOnes, kOnes, b0, b1);
      }
      // promote the group sums: R[0..1] row r0, R[2..3] row r1
      if constexpr (ASYM) {
        if constexpr (!MASK) {
#pragma unroll
          for (int i = 0; i < 4; ++i) Sg[i] = ac.S[i] - S0[i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const long long d = (long long)R[i] - (long long)tl.z[i >> 1] * (long long)Sg[i];
          ac.F[i] = fmaf(tl.c[i >> 1], (float)d, ac.F[i]);
        }
      } else if constexpr (RES) {
        ac.F[0] = fmaf(tl.c[0], (float)R[0], ac.F[0]);
        ac.F[1] = fmaf(tl.c[0], (float)R[1], ac.F[1]);
        ac.F[2] = fmaf(tl.c[1], (float)R[2], ac.F[2]);
        ac.F[3] = fmaf(tl.c[1], (float)R[3], ac.F[3]);
      }
      (void)S0;
      (void)Sg;
      if (EMIT) {
        const int ng = p.tpr;
        const int r0 = rb * kTileRows + gid, r1 = r0 + 8;
        const int a0 = tk0 + 8 * kg, a1 = tk1 + 8 * kg;
        if (a0 < p.M) {
          if (r0 < p.N) p.R_out[((int64_t)a0 * p.N + r0) * ng + cg] = R[0];
          if (r1 < p.N) p.R_out[((int64_t)a0 * p.N + r1) * ng + cg] = R[2];
        }
        if (a1 < p.M) {
          if (r0 < p.N) p.R_out[((int64_t)a1 * p.N + r0) * ng + cg] = R[1];
          if (r1 < p.N) p.R_out[((int64_t)a1 * p.N + r1) * ng + cg] = R[3];
        }
      }
    }
    // outlier channels of this tile (the same for every row): the lane
    // holding the channel forms the dequantized weight of its two rows;
    // the four lanes of its row group take it by shuffle
    const uint32_t om = omask[cg * 4 + tid4];
    uint32_t any = __ballot_sync(0xffffffffu, om != 0u) & 0xFu;  // lanes 0..3 = chunks 0..3
    while (any) {
      const int src = __ffs(any) - 1;
      any &= any - 1;
      uint32_t bits = __shfl_sync(0xffffffffu, om, src);
      int pos = __shfl_sync(0xffffffffu, obase[cg * 4 + tid4], src);
      const int owner = gid * 4 + src;
      while (bits) {
        const int j = __ffs(bits) - 1;
        bits &= bits - 1;
        float w0 = 0.0f, w1 = 0.0f, u0 = 0.0f, u1 = 0.0f;
        if (tid4 == src) {
          const int bit = tiled_bit_of(j);
          const uint32_t m0 = MASK ? (tl.m[0] >> bit) & 1u : 1u;
          const uint32_t m1 = MASK ? (tl.m[1] >> bit) & 1u : 1u;
          u0 = m0 ? (((tl.s[0] >> bit) & 1u) ? 1.0f : -1.0f) : 0.0f;
          u1 = m1 ? (((tl.s[1] >> bit) & 1u) ? 1.0f : -1.0f) : 0.0f;
          if constexpr (ASYM) {
            w0 = tl.c[0] * (float)(tile_code<0>(tl.q, j) - tl.z[0]);
            w1 = tl.c[1] * (float)(tile_code<1>(tl.q, j) - tl.z[1]);
          } else if constexpr (RES) {
            w0 = tl.c[0] * (float)tile_code<0>(tl.q, j);
            w1 = tl.c[1] * (float)tile_code<1>(tl.q, j);
          }
        }
        w0 = __shfl_sync(0xffffffffu, w0, owner);
        w1 = __shfl_sync(0xffffffffu, w1, owner);
        u0 = __shfl_sync(0xffffffffu, u0, owner);
        u1 = __shfl_sync(0xffffffffu, u1, owner);
        // (an index list that is not strictly ascending cannot push pos
        // past the list)
        if (pos >= 0 && pos < p.n_out) {
#pragma unroll
          for (int kg = 0; kg < NT; ++kg) {
            const int a0 = tk0 + 8 * kg, a1 = tk1 + 8 * kg;
            float x0, x1;
            if constexpr (FUSED) {
              x0 = a0 < p.M ? xo_s[a0 * p.n_pad + pos] : 0.0f;
              x1 = a1 < p.M ? xo_s[a1 * p.n_pad + pos] : 0.0f;
            } else {
              x0 = a0 < p.M ? __ldg(p.xout + (int64_t)a0 * p.n_out + pos) : 0.0f;
              x1 = a1 < p.M ? __ldg(p.xout + (int64_t)a1 * p.n_out + pos) : 0.0f;
            }
            Acc& ac = acc[kg];
            ac.Ut[0] = fmaf(u0, x0, ac.Ut[0]);
            ac.Ut[1] = fmaf(u0, x1, ac.Ut[1]);
            ac.Ut[2] = fmaf(u1, x0, ac.Ut[2]);
            ac.Ut[3] = fmaf(u1, x1, ac.Ut[3]);
            ac.Ur[0] = fmaf(w0, x0, ac.Ur[0]);
            ac.Ur[1] = fmaf(w0, x1, ac.Ur[1]);
            ac.Ur[2] = fmaf(w1, x0, ac.Ur[2]);
            ac.Ur[3] = fmaf(w1, x1, ac.Ur[3]);
          }
        }
        ++pos;
      }
    }

    // refill this slot with the tile D ahead, once no lane reads it
    __syncwarp();
    if (t + D < t1) copy_tile<MASK, RES, SPARSE, ASYM>(ring_u + slot_i * SL::kBytes, cur, lane);
    cp_async_commit();
    cur.advance<SPARSE, ASYM>();
    if (++slot_i == D) slot_i = 0;

    // end of a row block, or end of this warp's range
    if (cg == p.tpr - 1 || t + 1 == t1) {
#pragma unroll
      for (int kg = 0; kg < NT; ++kg) {
        const Acc& ac = acc[kg];
        const int a0 = tk0 + 8 * kg, a1 = tk1 + 8 * kg;
        float4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = cell(trunk_T<MASK>(ac, i), ac.F[i], ac.Ut[i], ac.Ur[i]);
        if (EMIT) {
          const int r0 = rb * kTileRows + gid, r1 = r0 + 8;
          if (a0 < p.M && r0 < p.N) atomicAdd(&p.T_out[(int64_t)a0 * p.N + r0], trunk_T<MASK>(ac, 0));
          if (a1 < p.M && r0 < p.N) atomicAdd(&p.T_out[(int64_t)a1 * p.N + r0], trunk_T<MASK>(ac, 1));
          if (a0 < p.M && r1 < p.N) atomicAdd(&p.T_out[(int64_t)a0 * p.N + r1], trunk_T<MASK>(ac, 2));
          if (a1 < p.M && r1 < p.N) atomicAdd(&p.T_out[(int64_t)a1 * p.N + r1], trunk_T<MASK>(ac, 3));
        }
        if (rb_head && cg == p.tpr - 1) {
          write_y(p, rb, gid, tid4, v, al0, al1, sx0[kg], sx1[kg], 8 * kg);
        } else {
          // a shared row block: slot 1 if this piece starts the row block
          // (this range ends inside it), slot 0 if it continues one begun
          // before this range
          const int slot = rb_head ? 1 : 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int tk = (i & 1) ? a1 : a0;
            if (tk < p.M) part_s[((warp * 2 + slot) * 16 + (i >> 1) * 8 + gid) * p.M + tk] = v[i];
          }
        }
      }
#pragma unroll
      for (int kg = 0; kg < NT; ++kg) acc_zero(acc[kg]);
      rb_head = true;
      if (cg == p.tpr - 1 && t + 1 < t1) {
        // the next row block starts: its row scales, needed at its end
        al0 = __ldg(p.alpha + (rb + 1) * kTileRows + gid);
        al1 = __ldg(p.alpha + (rb + 1) * kTileRows + gid + 8);
      }
    }
    if (++cg == p.tpr) {
      cg = 0;
      ++rb;
    }
  }

  // ---- row blocks shared by warps of this CTA ---------------------------------
  __syncthreads();
  if (t0 >= t1) return;
  // the row block whose first tile is in this warp's range and whose end lies
  // past it: this warp adds the parts of the CTA's later warps, in warp order
  // (al0 / al1 still hold its row scales)
  const int rb_last = (t1 - 1) / p.tpr;
  if (rb_last * p.tpr >= t0 && t1 % p.tpr != 0) {
    const int w_hi = tile_warp((rb_last + 1) * p.tpr - 1, T0c, T1c);
#pragma unroll
    for (int kg = 0; kg < NT; ++kg) {
      // (cells of tokens past M were never stored and are not written)
      auto cell_at = [&](int w, int slot, int i) -> const float4& {
        const int tk = min(((i & 1) ? tk1 : tk0) + 8 * kg, p.M - 1);
        return part_s[((w * 2 + slot) * 16 + (i >> 1) * 8 + gid) * p.M + tk];
      };
      float4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = cell_at(warp, 1, i);
      for (int w = warp + 1; w <= w_hi; ++w) {
        // a CTA with fewer tiles than warps has empty warps between its owners
        if (warp_first_tile(w, T0c, T1c) == warp_first_tile(w + 1, T0c, T1c)) continue;
#pragma unroll
        for (int i = 0; i < 4; ++i) cell_add(v[i], cell_at(w, 0, i));
      }
      write_y(p, rb_last, gid, tid4, v, al0, al1, sx0[kg], sx1[kg], 8 * kg);
    }
  }
}

template <bool MASK, bool EMIT, bool FUSED, int D, bool RES = true, bool SPARSE = false,
          bool ASYM = false, int NT = 1>
cudaError_t launch_one(const Params& p, int grid, int smem, bool pdl, cudaStream_t stream) {
  auto* fn = k_linear_tc<MASK, EMIT, FUSED, D, RES, SPARSE, ASYM, NT>;
  cudaError_t e = ensure_smem_attr((const void*)fn, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

// kind: 0 dense symmetric residual, 1 sparse, 2 asymmetric.
template <bool MASK, bool FUSED, int D, int NT>
cudaError_t launch_plain(const Params& p, bool res, int kind, int grid, int smem, bool pdl,
                         cudaStream_t stream) {
  if (!res)
    return launch_one<MASK, false, FUSED, kTrunkDepth, false, false, false, NT>(p, grid, smem, pdl,
                                                                               stream);
  if (kind == 1)
    return launch_one<MASK, false, FUSED, D, true, true, false, NT>(p, grid, smem, pdl, stream);
  if (kind == 2)
    return launch_one<MASK, false, FUSED, D, true, false, true, NT>(p, grid, smem, pdl, stream);
  return launch_one<MASK, false, FUSED, D, true, false, false, NT>(p, grid, smem, pdl, stream);
}

// Non-accumulator launch with a ring depth chosen at run time among Ds; two
// token groups (NT = 2) only from global codes (the fused split stages at
// most kCols tokens).
template <int D0, int... Ds>
cudaError_t launch_depth(int depth, bool mask, bool fused, bool res, int kind, int nt,
                         const Params& p, int grid, int smem, bool pdl, cudaStream_t stream) {
  if (depth == D0 || sizeof...(Ds) == 0) {
    if (fused)
      return mask ? launch_plain<true, true, D0, 1>(p, res, kind, grid, smem, pdl, stream)
                  : launch_plain<false, true, D0, 1>(p, res, kind, grid, smem, pdl, stream);
    if (nt == 2)
      return mask ? launch_plain<true, false, D0, 2>(p, res, kind, grid, smem, pdl, stream)
                  : launch_plain<false, false, D0, 2>(p, res, kind, grid, smem, pdl, stream);
    return mask ? launch_plain<true, false, D0, 1>(p, res, kind, grid, smem, pdl, stream)
                : launch_plain<false, false, D0, 1>(p, res, kind, grid, smem, pdl, stream);
  }
  if constexpr (sizeof...(Ds) > 0)
    return launch_depth<Ds...>(depth, mask, fused, res, kind, nt, p, grid, smem, pdl, stream);
  return cudaErrorInvalidValue;
}

// Accumulator-mode launch (two-tile ring).
template <int NT>
cudaError_t launch_emit(bool mask, int kind, const Params& p, int grid, int smem, bool pdl,
                        cudaStream_t stream) {
  if (kind == 1)
    return mask ? launch_one<true, true, false, kShallow, true, true, false, NT>(p, grid, smem, pdl, stream)
                : launch_one<false, true, false, kShallow, true, true, false, NT>(p, grid, smem, pdl, stream);
  if (kind == 2)
    return mask ? launch_one<true, true, false, kShallow, true, false, true, NT>(p, grid, smem, pdl, stream)
                : launch_one<false, true, false, kShallow, true, false, true, NT>(p, grid, smem, pdl, stream);
  return mask ? launch_one<true, true, false, kShallow, true, false, false, NT>(p, grid, smem, pdl, stream)
              : launch_one<false, true, false, kShallow, true, false, false, NT>(p, grid, smem, pdl, stream);
}

}  // namespace

size_t linear_tc_part_bytes(int) {
  // no row block is shared between CTAs: the workspace is not used
  return 0;
}

namespace {
// Partial sums of one token: kWarps warps x 2 slots x 16 rows.
constexpr int kSmemPartPerToken = kWarps * 2 * 16 * (int)sizeof(float4);
// Largest dynamic shared memory of one CTA on sm_100: 227 KiB (opt-in) less
// the kernel's static shared memory.
constexpr int kSmemMax = 227 * 1024 - 256;

int outlier_table_bytes(const sq_packed_weight& w) { return (int)(tiles_cols(w.K) / 32) * 8; }
int fused_token_bytes(const sq_packed_weight& w, int n_out) {
  return (int)tiles_cols(w.K) + (int)round_up(n_out, 4) * 4;
}
// kind: 0 dense symmetric residual, 1 sparse, 2 asymmetric.
int ring_bytes(bool mask, int depth, int kind = 0) {
  int slot;
  if (kind == 1) slot = mask ? Slot<true, true, true>::kBytes : Slot<false, true, true>::kBytes;
  else if (kind == 2) slot = mask ? Slot<true, true, false, true>::kBytes : Slot<false, true, false, true>::kBytes;
  else slot = mask ? Slot<true>::kBytes : Slot<false>::kBytes;
  return kWarps * depth * slot;
}
int residual_kind(const sq_packed_weight& w) {
  return w.layout == SQ_LAYOUT_TILES_SPARSE ? 1 : w.layout == SQ_LAYOUT_TILES_ASYM ? 2 : 0;
}
int trunk_ring_bytes(bool mask) {
  return kWarps * kTrunkDepth * (mask ? Slot<true, false>::kBytes : Slot<false, false>::kBytes);
}
}  // namespace

int linear_tc_pass_tokens(const sq_packed_weight& w, bool trunk_only) {
  // two token groups per pass where 2 kCols tokens' partial sums fit beside
  // the shallow ring (every shape whose outlier table is small enough)
  const int ring = trunk_only ? trunk_ring_bytes(w.mask_bits != nullptr)
                              : ring_bytes(w.mask_bits != nullptr, kShallow, residual_kind(w));
  const int need = kSmemPartPerToken * 2 * kCols + outlier_table_bytes(w) + 16 + ring;
  return need <= kSmemMax ? 2 * kCols : kCols;
}

int linear_tc_fused_tokens(const sq_packed_weight& w, int n_out) {
  // counted with the shallow ring; the deep one is used when it fits
  const int fixed = ring_bytes(w.mask_bits != nullptr, kShallow, residual_kind(w)) +
                    outlier_table_bytes(w) +
                    kCols * 4 + kWarps * kCols * 4 + 64;
  const int per = fused_token_bytes(w, n_out) + kSmemPartPerToken;
  const int m = (kSmemMax - fixed) / per;
  return m < 0 ? 0 : std::min(m, kCols);
}

cudaError_t launch_linear_tc(const sq_packed_weight& w, int M, const int8_t* xq, const float* sx,
                             const float* x_out, const float* x, const int32_t* idx, int n_out,
                             float* y, int32_t* T_out, int32_t* R_out, void* workspace,
                             size_t part_bytes, int sm_count, int32_t* status, bool pdl,
                             bool trunk_only, cudaStream_t stream) {
  const int kind = residual_kind(w);
  const bool sparse = kind == 1;
  if (M < 1 || M > linear_tc_pass_tokens(w, trunk_only)) return cudaErrorInvalidValue;
  if (w.layout != SQ_LAYOUT_TILES && w.layout != SQ_LAYOUT_TILES_SPARSE &&
      w.layout != SQ_LAYOUT_TILES_ASYM)
    return cudaErrorInvalidValue;
  if (sparse && (!w.keep_bits || !w.res_bytes)) return cudaErrorInvalidValue;
  if (kind == 2 && !w.res_zero) return cudaErrorInvalidValue;
  if (trunk_only && T_out) return cudaErrorInvalidValue;
  const bool fused = x != nullptr;
  if (fused && (T_out || M > linear_tc_fused_tokens(w, n_out))) return cudaErrorInvalidValue;
  const int nt = M > kCols ? 2 : 1;
  Params p;
  p.res = w.res_q;
  p.sign = w.sign_bits;
  p.mask = w.mask_bits;
  p.alpha = w.alpha;
  p.scale = w.res_scale;
  p.keep = w.keep_bits;
  p.nbytes = w.res_bytes;
  p.zero = w.res_zero;
  p.N = w.N;
  p.K = w.K;
  p.tpr = (int)(tiles_cols(w.K) / kTileK);
  const int64_t T = ceil_div(w.N, kTileRows) * (int64_t)p.tpr;
  if (T >= INT32_MAX / 2) return cudaErrorInvalidValue;
  p.T = (int)T;
  p.n_rb = (int)ceil_div(w.N, kTileRows);
  // The fewest CTAs with the largest share of row blocks that one CTA per SM
  // gives: every CTA then streams the same number of row blocks (qkv: 128 x 6
  // instead of 28 x 6 + 120 x 5) and none of them finishes alone with the
  // memory system idle around it (7B-shaped stack on B200: 3798 -> 3896 GB/s).
  const int64_t cap = std::max<int64_t>(1, std::min<int64_t>((int64_t)sm_count * kBps, p.n_rb));
  const int64_t share = (p.n_rb + cap - 1) / cap;
  const int64_t blocks = std::max<int64_t>(1, (p.n_rb + share - 1) / share);
  p.M = M;
  p.xq = xq;
  p.xs = (int)xq_stride_of(w.K);
  p.sx = sx;
  p.xout = x_out;
  p.idx = idx;
  p.n_out = n_out;
  p.y = y;
  p.T_out = T_out;
  p.R_out = R_out;
  (void)workspace;
  (void)part_bytes;
  p.pdl = pdl ? 1 : 0;
  p.x = x;
  p.status = status;
  p.n_pad = (int)round_up(n_out, 4);
  const bool mask = w.mask_bits != nullptr;
  const bool emit = T_out != nullptr;
  int smem = kSmemPartPerToken * M;
  p.off_omask = smem;
  smem += outlier_table_bytes(w);
  p.off_xq = p.off_xo = p.off_sx = p.off_red = 0;
  if (fused) {
    p.off_xq = smem;
    smem += M * p.xs;
    p.off_xo = smem;
    smem += M * p.n_pad * 4;
    p.off_sx = smem;
    smem += kCols * 4;
    p.off_red = smem;
    smem += kWarps * kCols * 4;
  }
  smem = (int)round_up(smem, 16);
  p.off_ring = smem;
  // three tiles per warp above batch 2 where they fit, else two (the
  // accumulator mode, used to check the kernel, always takes two)
  const int depth =
      (!emit && M > 2 && smem + ring_bytes(mask, kDeep, kind) <= kSmemMax) ? kDeep : kShallow;
  smem += trunk_only ? trunk_ring_bytes(mask) : ring_bytes(mask, depth, kind);
  if (smem > kSmemMax) return cudaErrorInvalidValue;
  const int grid = (int)blocks;
  if (emit)
    return nt == 2 ? launch_emit<2>(mask, kind, p, grid, smem, pdl, stream)
                   : launch_emit<1>(mask, kind, p, grid, smem, pdl, stream);
  return launch_depth<kDeep, kShallow>(depth, mask, fused, !trunk_only, kind, nt, p, grid, smem,
                                       pdl, stream);
}

}  // namespace sq
