// sq_nvfp4.cu -- the prefill path of format separation: NVFP4 weights and
// activations multiplied on the 5th-generation tensor cores with block
// scaling (tcgen05.mma kind::mxf4nvf4, 16-element UE4M3 scales).
//
// Page: the ISTA-DASLab news page on separated quantization (paragraphs 2-4):
// prefill uses the hardware's native quantized compute (NVFP4) while decode
// keeps its own low-bit weight-only format.  The page names the format
// without defining it; the reading taken is the format the Blackwell tensor
// cores consume:
//   E2M1 elements (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; sign in bit 3; two
//   per byte, the lower channel in the low nibble), blocks of 16 channels with
//   one UE4M3 scale s_b, and a binary32 second-level scale g = amax / (6*448)
//   per weight tensor and per activation row (token).
//   s_b = RNE_ue4m3(amax_b / (6 g)), q = RNE_e2m1(x / (s_b g)) saturating at
//   6, ties to the even code, +0 for a zero result; g = 0 or s_b = 0 -> 0.
//   y[t][n] = g_w g_x[t] sum_b s_w[n][b] s_x[t][b] sum_{j in b} e(qw) e(qx).
//
// Quantizer decisions are exact: the block scale rounds the binary64
// quotient amax_b / (6 g) (6 g is exact in binary64, and a quotient of a
// 24-bit by a 26-bit significand that is not a rounding midpoint lies more
// than 2^-32 of itself from one, far beyond binary64 rounding); the element
// code compares |x| with the seven E2M1 midpoints times s_b g, each product
// exact in binary64.
//
// GEMM: a persistent kernel, one CTA per SM, looping over output tiles of
// 128 tokens (MMA M, one TMEM lane each) x 192 weight rows (MMA N), token
// tiles fastest so that concurrent CTAs share weight tiles in L2.  Stages of
// 256 channels (128 bytes a row, 128-byte swizzle) run through a 4-stage
// ring without draining between tiles.
//   warp 0 (one lane): TMA of both code tiles, bulk copies of the scale
//     chunks (2 KB for the tokens, 2 x 2 KB for the two 128-row scale blocks
//     the weight tile lies in) into the ring;
//   warps 6-9 (one per tensor-memory lane quarter): per stage, the scales
//     from shared memory into one of two scale sets of tensor memory
//     (tcgen05.st, every quarter holding all of them: lane i of quarter q,
//     word c = the scales of row 32 c + i; set g % 2, written once the MMAs
//     of stage g - 2 are done), then arrive on the stage's scale barrier;
//   warp 1 (one lane): per stage, 4 block-scaled MMAs (K = 64 each) into one
//     of two fp32 accumulators (tiles alternate);
//   warps 2-5: read an accumulator back (tcgen05.ld), free it for the tile
//     after next, scale by g_w g_x[t], and stage y in shared memory in 32 x 32
//     blocks that leave through tensor stores (else through stores of whole
//     128-byte row segments; each thread storing its own row measured 117
//     against 89 us).
// Shared-memory bandwidth is the budget the roles share: per stage the copies
// write 46 KB, the MMAs read 40 KB and the four scale warps each read the
// stage's scales (16-byte loads: 4-byte loads at a 16-byte lane stride cost
// four times the wavefronts and the launch 92 against 86 us).
// The scales go in through the warps rather than tcgen05.cp: eight copies
// per stage issued beside the MMAs took 131 us against 95 us per launch at
// 2048 x 4096 -> 14336 (then with 128-row weight tiles; 192 rows took the
// launch from 99.9 to 94.0 us on one box: fewer shared-memory bytes per MAC).
// Tensor memory: accumulators at columns [0,192) and [192,384), the scale
// sets at 384 and 432 (A 16 columns, then B 32).  Every wait is bounded: a
// wait that runs out sets SQ_ERR_TIMEOUT and the CTA drains its copies and
// MMAs before it frees its tensor memory.
#include <stdint.h>

#include <algorithm>

#include "sq_internal.h"
#include "sq_tcgen05.cuh"

namespace sq {
namespace {

using tc05::fence_after;
using tc05::fence_before;

constexpr int BM = 128;          // tokens per tile (MMA M)
constexpr int BN = 192;          // weight rows per tile (MMA N)
constexpr int kStageK = 256;     // channels per stage
constexpr int kRowBytes = kStageK / 2;  // code bytes per row per stage
constexpr int kStages = 4;
constexpr int kThreads = 320;    // 10 warps
constexpr uint32_t kTmemCols = 512;
// tensor memory: accumulator b at columns [192 b, 192 b + 192); the scales of
// stage g in set g % 2 at kSfCol0 + 48 (g % 2): A 16 columns, then B 32
// (eight 32-row words per 64-channel chunk, as for 256 rows; words 6-7 zero)
constexpr uint32_t kSfCol0 = 2 * BN;
constexpr uint32_t kSfSet = 48;

constexpr int kBytesA = BM * kRowBytes;  // 16 KB
constexpr int kBytesB = BN * kRowBytes;  // 24 KB
constexpr int kBytesSf = 4 * 512;        // one 128-row block: 4 chunks of 128 rows x 4 scales
// the weight tile's 192 rows start at a multiple of 64 and lie in two
// consecutive 128-row scale blocks
constexpr int kOffA = 0, kOffB = kBytesA, kOffSa = kOffB + kBytesB, kOffSb = kOffSa + kBytesSf;
constexpr int kStageBytes = kOffSb + 2 * kBytesSf;  // 46 KB
static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
static_assert(kSfCol0 + 2 * kSfSet <= kTmemCols, "scale columns past the allocation");
static_assert(BN % 64 == 0 && BN <= 192, "tiles start at 0 or 64 in a scale block and end in the next");
// y staging for the epilogue, per warp: two 32 x 32 float blocks in the
// 128-byte-swizzled layout of a tensor store (16-byte chunk j of row r at
// chunk j ^ (r % 8), so the 16-byte stores of 8 consecutive lanes hit distinct
// banks); without the tensor store, one block with rows 36 floats apart.
constexpr int kStageRow = 36;
constexpr int kOffOut = kStages * kStageBytes;
constexpr int kOutBlock = 32 * 32 * 4;         // 4 KB, 1024-byte aligned
constexpr int kOutBytes = 4 * 2 * kOutBlock;   // 32 KB
static_assert(kOffOut % 1024 == 0, "swizzled staging must be 1024-byte aligned");
static_assert(4 * 32 * kStageRow * 4 <= kOutBytes, "padded staging past its area");

struct Aux {
  uint64_t full[kStages], empty[kStages], sfr[kStages], accf[2], acce[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr int kSmemBytes = kOffOut + kOutBytes + (int)sizeof(Aux) + 1024;

struct Params {
  int M, N, nk;   // nk = stages per tile = K256 / 256
  int nt_m, tiles;
  int sf_chunks;  // 64-channel scale chunks per 128-row block
  int nblk_b;     // 128-row scale blocks of the weight
  const uint8_t* sfa;  // activation scale chunks
  const uint8_t* sfb;  // weight scale chunks
  const float* gx;     // [M]
  const float* gw;     // [1]
  float* y;
  int32_t* status;
  uint64_t wait_ns;
  int skip_stage;  // failure injection for tests: this stage is never requested (-1: none)
};

// D (f32) += A (E2M1, K-major) * B (E2M1, K-major) with UE4M3 block scales
// of 16; M = 128, N = 192, K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t sfa,
                                        uint32_t sfb, bool acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(acc ? 1 : 0), "r"(sfa), "r"(sfb));
}

// 16 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}

// 32 consecutive TMEM columns of this thread's lane (waits for both stores).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&w)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15]),
      "r"(w[16]), "r"(w[17]), "r"(w[18]), "r"(w[19]), "r"(w[20]), "r"(w[21]), "r"(w[22]), "r"(w[23]),
      "r"(w[24]), "r"(w[25]), "r"(w[26]), "r"(w[27]), "r"(w[28]), "r"(w[29]), "r"(w[30]), "r"(w[31])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Aux* aux,
                                              const Params& p) {
  if (mbar_wait(bar, parity, p.wait_ns)) return true;
  set_status(p.status, SQ_ERR_TIMEOUT);
  atomicExch(&aux->abort, 1);
  return false;
}
__device__ __forceinline__ bool aborted(const Aux* aux) {
  return *reinterpret_cast<const volatile int*>(&aux->abort) != 0;
}

// TMA_Y: y leaves through tensor stores of the staged 32 x 32 blocks (y
// 16-byte aligned and N % 4 = 0), else through 16-byte stores of whole
// 128-byte row segments.
template <bool TMA_Y>
__global__ void __launch_bounds__(kThreads, 1)
    k_nvfp4_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmY, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Aux* aux = reinterpret_cast<Aux*>(smem + kOffOut + kOutBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&aux->full[s], 1);
      mbar_init(&aux->empty[s], 1);
      mbar_init(&aux->sfr[s], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&aux->accf[b], 1);
      mbar_init(&aux->acce[b], 128);
    }
    mbar_init(&aux->drain, 1);
    aux->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tc05::tmem_alloc(&aux->tmem_base, kTmemCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = aux->tmem_base;

  if (warp == 0) {
    // ---- producer: every stage of every tile of this CTA, in order
    if (lane == 0) {
      int last_use[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) last_use[s] = -1;
      uint32_t g = 0;  // stages issued so far
      for (int tile = blockIdx.x; tile < p.tiles && !aborted(aux); tile += gridDim.x) {
        const int mt = tile % p.nt_m, nt = tile / p.nt_m;
        const int cb0 = (nt * BN) >> 7;  // first 128-row scale block of the tile
        const bool two = cb0 + 1 < p.nblk_b;
        const uint8_t* sfa = p.sfa + (int64_t)mt * p.sf_chunks * 512;
        const uint8_t* sfb = p.sfb + (int64_t)cb0 * p.sf_chunks * 512;
        for (int kb = 0; kb < p.nk; ++kb, ++g) {
          const int s = (int)(g % kStages);
          const uint32_t use = g / kStages;
          if (g >= kStages && !wait_or_abort(&aux->empty[s], (use & 1u) ^ 1u, aux, p)) break;
          if (aborted(aux)) break;
          if (kb == p.skip_stage) continue;  // (tests only) never requested: its waits run out
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&aux->full[s], kStageBytes - (two ? 0 : kBytesSf));
          tc05::tma_load_2d(st + kOffA, &tmA, kb * kRowBytes, mt * BM, &aux->full[s]);
          tc05::tma_load_2d(st + kOffB, &tmB, kb * kRowBytes, nt * BN, &aux->full[s]);
          tc05::bulk_load(st + kOffSa, sfa + (int64_t)kb * kBytesSf, kBytesSf, &aux->full[s]);
          tc05::bulk_load(st + kOffSb, sfb + (int64_t)kb * kBytesSf, kBytesSf, &aux->full[s]);
          if (two)
            tc05::bulk_load(st + kOffSb + kBytesSf, sfb + ((int64_t)p.sf_chunks + 4 * kb) * 512,
                            kBytesSf, &aux->full[s]);
          last_use[s] = (int)use;
        }
      }
      // winding down after a timeout: every requested stage must have landed
      if (aborted(aux)) {
#pragma unroll
        for (int s = 0; s < kStages; ++s)
          if (last_use[s] >= 0) (void)mbar_wait(&aux->full[s], (uint32_t)last_use[s] & 1u, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---- scale copies and MMAs
    if (lane == 0) {
      uint32_t g = 0, n = 0;  // stages consumed, tiles started
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++n) {
        const uint32_t b = n & 1u;
        if (n >= 2 && !wait_or_abort(&aux->acce[b], ((n >> 1) & 1u) ^ 1u, aux, p)) break;
        fence_after();
        const uint32_t d = tmem + BN * b;
        bool ok = true;
        for (int kb = 0; kb < p.nk; ++kb, ++g) {
          const int s = (int)(g % kStages);
          if (!wait_or_abort(&aux->full[s], (g / kStages) & 1u, aux, p) ||
              !wait_or_abort(&aux->sfr[s], (g / kStages) & 1u, aux, p)) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t st = smem_u32(smem + s * kStageBytes);
          const uint32_t ta = tmem + kSfCol0 + kSfSet * (g & 1u), tb = ta + 16;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_fp4(d, tc05::sw128_desc(st + kOffA + 32 * kk), tc05::sw128_desc(st + kOffB + 32 * kk),
                    ta + 4 * kk, tb + 8 * kk, kb > 0 || kk > 0);
          tc05::mma_commit(&aux->empty[s]);
        }
        if (!ok) break;
        tc05::mma_commit(&aux->accf[b]);
      }
      // winding down after a timeout: the MMAs issued must be done before the
      // tensor memory is freed
      if (aborted(aux)) {
        tc05::mma_commit(&aux->drain);  // tracks every MMA and copy issued before it
        (void)mbar_wait(&aux->drain, 0u, p.wait_ns);
      }
    }
  } else if (warp >= 6) {
    // ---- scale factors into tensor memory: this warp's lane quarter, in
    // set g % 2 once the MMAs of stage g - 2 (the set's last readers) are done
    const int q = warp & 3;
    uint32_t g = 0;
    for (int tile = blockIdx.x; tile < p.tiles && !aborted(aux); tile += gridDim.x) {
      const int n0 = (tile / p.nt_m) * BN;
      const int cb0 = n0 >> 7;
      const bool two = cb0 + 1 < p.nblk_b;
      const bool shifted = (n0 & 127) != 0;  // n0 % 128 is 0 or 64
      bool ok = true;
      for (int kb = 0; kb < p.nk; ++kb, ++g) {
        const int s = (int)(g % kStages);
        ok = wait_or_abort(&aux->full[s], (g / kStages) & 1u, aux, p) &&
             (g < 2 || wait_or_abort(&aux->empty[(g - 2) % kStages], ((g - 2) / kStages) & 1u, aux, p));
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint8_t* st = smem + s * kStageBytes;
        // Each lane reads its 16 bytes of every chunk (a 128-row block's four
        // 32-row words for one 64-channel chunk) with one vector load; the
        // tile's words are picked in registers.  Four-byte loads at a 16-byte
        // lane stride would hit each bank four times, and the four warps'
        // reads share the bandwidth with the copies and the MMAs.
        uint32_t wa[16], wb[32];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint4 a = *reinterpret_cast<const uint4*>(st + kOffSa + 512 * kk + 16 * lane);
          wa[4 * kk] = a.x;
          wa[4 * kk + 1] = a.y;
          wa[4 * kk + 2] = a.z;
          wa[4 * kk + 3] = a.w;
          const uint4 b0 = *reinterpret_cast<const uint4*>(st + kOffSb + 512 * kk + 16 * lane);
          const uint4 b1 = two ? *reinterpret_cast<const uint4*>(st + kOffSb + kBytesSf + 512 * kk + 16 * lane)
                               : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t w[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
          // tile row 32 j + lane is word j of the two blocks' words, or word
          // j + 2 when the tile starts 64 rows into its first block
#pragma unroll
          for (int j = 0; j < 8; ++j)
            wb[8 * kk + j] = j < BN / 32 ? (shifted ? w[j + 2] : w[j]) : 0u;
        }
        const uint32_t ts = tmem + ((uint32_t)(32 * q) << 16) + kSfCol0 + kSfSet * (g & 1u);
        tmem_st16(ts, wa);
        tmem_st32(ts + 16, wb);
        fence_before();
        mbar_arrive(&aux->sfr[s]);
      }
      if (!ok) break;
    }
  } else {
    // ---- epilogue: one token (TMEM lane) per thread
    const int q = warp & 3;  // TMEM lane quarter of this warp
    float* stage_out = reinterpret_cast<float*>(smem + kOffOut) + q * 32 * kStageRow;
    uint8_t* blocks = smem + kOffOut + q * 2 * kOutBlock;  // TMA_Y: this warp's two blocks
    uint32_t nb = 0;                                       // blocks stored so far
    const float gw = __ldg(p.gw);
    uint32_t n = 0;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++n) {
      const uint32_t b = n & 1u;
      const int m0 = (tile % p.nt_m) * BM + 32 * q, n0 = (tile / p.nt_m) * BN;
      bool ok = !aborted(aux) && wait_or_abort(&aux->accf[b], (n >> 1) & 1u, aux, p);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      fence_after();
      const int t = m0 + lane;
      const float sc = (t < p.M ? __ldg(p.gx + t) : 0.0f) * gw;
#pragma unroll 1
      for (int h = 0; h < BN / 32; ++h) {
        int r[32];
        tc05::tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + BN * b + 32 * h, r);
        if (h == BN / 32 - 1) {
          fence_before();
          mbar_arrive(&aux->acce[b]);
        }
        if constexpr (TMA_Y) {
          const int x0 = n0 + 32 * h;
          if (m0 >= p.M || x0 >= p.N) continue;  // the whole block is outside y
          uint8_t* blk = blocks + (nb & 1u) * kOutBlock;
          // the store that last read this block (two blocks ago) is done reading
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(blk + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_float4(sc * __int_as_float(r[4 * j]), sc * __int_as_float(r[4 * j + 1]),
                            sc * __int_as_float(r[4 * j + 2]), sc * __int_as_float(r[4 * j + 3]));
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            // rows past M and columns past N are clipped by the tensor store
            asm volatile(
                "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                    reinterpret_cast<uint64_t>(&tmY)),
                "r"(x0), "r"(m0), "r"(smem_u32(blk))
                : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
          ++nb;
        } else {
          // this lane's row of the 32 x 32 block into shared memory
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(stage_out + lane * kStageRow + i) =
                make_float4(sc * __int_as_float(r[i]), sc * __int_as_float(r[i + 1]),
                            sc * __int_as_float(r[i + 2]), sc * __int_as_float(r[i + 3]));
          __syncwarp();
          // four rows per store: lanes 8j .. 8j+7 write row 4i + j, 128 bytes
          const int cn = n0 + 32 * h + 4 * (lane & 7);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = 4 * i + (lane >> 3);
            const int tt = m0 + rr;
            const float4 v = *reinterpret_cast<const float4*>(stage_out + rr * kStageRow + 4 * (lane & 7));
            if (tt < p.M) {
              float* yp = p.y + (int64_t)tt * p.N + cn;
              if (cn + 4 <= p.N && (p.N & 3) == 0) {
                *reinterpret_cast<float4*>(yp) = v;
              } else {
                if (cn < p.N) yp[0] = v.x;
                if (cn + 1 < p.N) yp[1] = v.y;
                if (cn + 2 < p.N) yp[2] = v.z;
                if (cn + 3 < p.N) yp[3] = v.w;
              }
            }
          }
          __syncwarp();
        }
      }
    }
    // the tensor stores have written y before the CTA leaves
    if (TMA_Y && lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tc05::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- quantizers ------------------------------------------------------------------

// Nearest UE4M3 code of q >= 0 (a binary64 value), ties to the even code,
// saturating at 448 (code 126).
__device__ __forceinline__ uint32_t ue4m3_rne(double q) {
  if (!(q > 0.0)) return 0u;
  if (q >= 448.0) return 126u;
  if (q < 0.015625) return (uint32_t)rint(q * 512.0);  // subnormals m * 2^-9 (8 = 2^-6)
  const uint64_t bits = (uint64_t)__double_as_longlong(q);
  int e = (int)((bits >> 52) & 0x7FF) - 1023;  // -6 .. 8
  const uint64_t man = bits & ((1ull << 52) - 1);
  uint32_t m = (uint32_t)(man >> 49);
  const uint64_t rem = man & ((1ull << 49) - 1), half = 1ull << 48;
  if (rem > half || (rem == half && (m & 1u))) ++m;
  if (m == 8u) {
    m = 0u;
    ++e;
  }
  const uint32_t code = ((uint32_t)(e + 7) << 3) | m;
  return code > 126u ? 126u : code;
}

__device__ __forceinline__ double ue4m3_val(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  if (e == 0u) return (double)m * 0x1p-9;
  // (1 + m/8) * 2^(e-7) from its binary64 fields
  return __longlong_as_double((long long)(((uint64_t)(e - 7u + 1023u) << 52) | ((uint64_t)m << 49)));
}

// E2M1 code of x against the step s_b * g: the number of midpoints below
// |x| (a midpoint reached exactly counts when the code above it is even).
struct E2m1Thresholds {
  double t[7];
};
__device__ __forceinline__ E2m1Thresholds e2m1_thresholds(double step) {
  E2m1Thresholds th;
  th.t[0] = 0.25 * step;
  th.t[1] = 0.75 * step;
  th.t[2] = 1.25 * step;
  th.t[3] = 1.75 * step;
  th.t[4] = 2.5 * step;
  th.t[5] = 3.5 * step;
  th.t[6] = 5.0 * step;
  return th;
}
__device__ __forceinline__ uint32_t e2m1_code(float x, const E2m1Thresholds& th) {
  const double a = fabs((double)x);
  uint32_t c = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) c += (i & 1) ? (a >= th.t[i] ? 1u : 0u) : (a > th.t[i] ? 1u : 0u);
  return (c != 0u && x < 0.0f) ? (c | 8u) : c;
}

// Byte offset of the scale of (row r, 16-channel block b) in the chunked
// layout: chunk (r / 128, b / 4) of 512 bytes, then row r % 32 at 16 bytes,
// word (r % 128) / 32, byte b % 4.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t b, int sf_chunks) {
  return ((r >> 7) * sf_chunks + (b >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (b & 3);
}

__device__ __forceinline__ float absmax_reduce(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  v = red[0];
  __syncthreads();
  return v;
}

// amax of a whole tensor: atomicMax on the bit pattern of |x| (non-negative
// floats order like their bits).  Non-finite entries set SQ_ERR_NONFINITE.
__global__ void k_nvfp4_amax(const float* __restrict__ X, int64_t n, uint32_t* amax_bits,
                             int32_t* status) {
  __shared__ float red[32];
  float a = 0.0f;
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = __ldg(X + i);
    if (!isfinite(v)) bad = true;
    a = fmaxf(a, fabsf(v));
  }
  if (bad) set_status(status, SQ_ERR_NONFINITE);
  a = absmax_reduce(a, red);
  if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(a));
}

// E2M1 code of x given the block's step s_b g: a binary32 estimate
// u = |x| * (4 / step) (relative error below 3 * 2^-24) decides unless u lies
// within 2^-19 of one of the seven midpoints (4 x 0.25, 0.75, 1.25, 1.75, 2.5,
// 3.5, 5 = 1, 3, 5, 7, 10, 14, 20); then the exact binary64 comparison
// decides.  Away from them the code is the number of midpoints at or below
// floor(u), one popcount.
__device__ __forceinline__ uint32_t e2m1_code_fast(float x, float inv4, double step) {
  const float u = fabsf(x) * inv4;
  const float uc = fminf(u, 31.0f);
  const float r = rintf(uc);
  constexpr uint32_t kMid4 = (1u << 1) | (1u << 3) | (1u << 5) | (1u << 7) | (1u << 10) | (1u << 14) |
                             (1u << 20);
  if (((kMid4 >> (uint32_t)r) & 1u) && fabsf(u - r) <= u * 0x1p-19f)
    return e2m1_code(x, e2m1_thresholds(step));
  const uint32_t k = (uint32_t)uc;  // floor: uc >= 0
  const uint32_t c = (uint32_t)__popc(kMid4 & ((2u << k) - 1u));
  return (c != 0u && x < 0.0f) ? (c | 8u) : c;
}

// The codes (two words, channel 2i in the low nibble of byte i) and the
// scale code of one 16-channel block under second-level scale g.
__device__ __forceinline__ uint32_t quantize_block(const float (&v)[16], float gr, uint2& out) {
  float ab = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) ab = fmaxf(ab, fabsf(v[i]));
  const double gd = (double)gr;
  const uint32_t sc = gr == 0.0f ? 0u : ue4m3_rne((double)ab / (6.0 * gd));
  const double step = ue4m3_val(sc) * gd;
  uint32_t w0 = 0u, w1 = 0u;
  if (step != 0.0) {
    const float inv4 = 4.0f * __frcp_rn(__double2float_rn(step));
#pragma unroll
    for (int i = 0; i < 8; ++i) w0 |= e2m1_code_fast(v[i], inv4, step) << (4 * i);
#pragma unroll
    for (int i = 0; i < 8; ++i) w1 |= e2m1_code_fast(v[8 + i], inv4, step) << (4 * i);
  }
  out = make_uint2(w0, w1);
  return sc;
}

__device__ __forceinline__ void load_block(const float* x, int j0, int K, bool live, float (&v)[16]) {
  if (live && j0 + 16 <= K && (K & 3) == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(x + j0) + i);
      v[4 * i] = f.x;
      v[4 * i + 1] = f.y;
      v[4 * i + 2] = f.z;
      v[4 * i + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = (live && j0 + i < K) ? __ldg(x + j0 + i) : 0.0f;
  }
}

// One CTA per row (rows_pad of them): every 16-channel block of the row up to
// K256.  PER_ROW: g from the row's own amax (written to g[r]); else g from
// the tensor amax in amax_bits (written to g[0] by CTA 0).  BPT > 0: each
// thread holds its BPT blocks in registers between the amax and the codes
// (one read of the row); BPT = 0: any K, the row is read twice.
template <bool PER_ROW, int BPT>
__global__ void __launch_bounds__(512) k_nvfp4_quantize(const float* __restrict__ X, int rows, int K,
                                                        int code_stride, int sf_chunks,
                                                        uint8_t* __restrict__ codes,
                                                        uint8_t* __restrict__ scales, float* g,
                                                        const uint32_t* amax_bits, int32_t* status) {
  __shared__ float red[32];
  const int r = blockIdx.x;
  const bool live = r < rows;
  const float* x = X + (int64_t)(live ? r : 0) * K;
  const int nb = code_stride / 8;  // 16-channel blocks up to K256
  constexpr int kHeld = BPT > 0 ? BPT : 1;
  float v[kHeld][16];
  float a = 0.0f;
  bool bad = false;
  if constexpr (BPT > 0) {
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int b = threadIdx.x + i * blockDim.x;
      load_block(x, 16 * b, K, live && b < nb, v[i]);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if (!isfinite(v[i][e])) bad = true;
        a = fmaxf(a, fabsf(v[i][e]));
      }
    }
  } else if (PER_ROW && live) {
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      const float t = __ldg(x + j);
      if (!isfinite(t)) bad = true;
      a = fmaxf(a, fabsf(t));
    }
  }
  float gr;
  if (PER_ROW) {
    if (bad) set_status(status, SQ_ERR_NONFINITE);
    a = absmax_reduce(a, red);
    gr = live ? __double2float_rn((double)a / 2688.0) : 0.0f;
    if (threadIdx.x == 0) g[r] = gr;
  } else {
    gr = __double2float_rn((double)__uint_as_float(*amax_bits) / 2688.0);
    if (r == 0 && threadIdx.x == 0) g[0] = gr;
  }
  uint8_t* crow = codes + (int64_t)r * code_stride;
  if constexpr (BPT > 0) {
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int b = threadIdx.x + i * blockDim.x;
      if (b < nb) {
        uint2 w;
        const uint32_t sc = quantize_block(v[i], gr, w);
        *reinterpret_cast<uint2*>(crow + 8 * b) = w;
        scales[sf_offset(r, b, sf_chunks)] = (uint8_t)sc;
      }
    }
  } else {
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
      load_block(x, 16 * b, K, live, v[0]);
      uint2 w;
      const uint32_t sc = quantize_block(v[0], gr, w);
      *reinterpret_cast<uint2*>(crow + 8 * b) = w;
      scales[sf_offset(r, b, sf_chunks)] = (uint8_t)sc;
    }
  }
}

template <bool PER_ROW>
cudaError_t launch_quantize_rows(const float* X, const sq_nvfp4_matrix& out, const uint32_t* amax,
                                 int32_t* status, cudaStream_t stream) {
  const int nb = out.code_stride / 8;
  const int threads = nb <= 128 ? 128 : (nb <= 256 ? 256 : 512);
  const int bpt = (nb + threads - 1) / threads;
  auto go = [&](auto kern) {
    kern<<<out.rows_pad, threads, 0, stream>>>(X, out.rows, out.K, out.code_stride, out.sf_chunks,
                                               out.codes, out.scales, out.g, amax, status);
    return cudaGetLastError();
  };
  if (bpt == 1) return go(k_nvfp4_quantize<PER_ROW, 1>);
  if (bpt == 2) return go(k_nvfp4_quantize<PER_ROW, 2>);
  if (bpt <= 4) return go(k_nvfp4_quantize<PER_ROW, 4>);
  return go(k_nvfp4_quantize<PER_ROW, 0>);
}

}  // namespace

cudaError_t launch_nvfp4_quantize(const float* X, const sq_nvfp4_matrix& out, int32_t* status,
                                  cudaStream_t stream) {
  if (out.per_row) return launch_quantize_rows<true>(X, out, nullptr, status, stream);
  uint32_t* amax = reinterpret_cast<uint32_t*>(out.g + 1);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  const int64_t n = (int64_t)out.rows * out.K;
  const int64_t want = (n + 255) / 256;
  const int grid = (int)(want < 4096 ? want : 4096);
  k_nvfp4_amax<<<grid, 256, 0, stream>>>(X, n, amax, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_quantize_rows<false>(X, out, amax, status, stream);
}

cudaError_t launch_nvfp4_gemm(const sq_nvfp4_matrix& w, const sq_nvfp4_matrix& x, float* y,
                              int32_t* status, cudaStream_t stream, uint64_t wait_ns,
                              int skip_stage) {
  if (w.K != x.K || w.code_stride != x.code_stride || w.per_row || !x.per_row)
    return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (!tc05::make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, x.codes, (uint64_t)x.code_stride,
                      (uint64_t)x.rows_pad, (uint64_t)x.code_stride, kRowBytes, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tc05::make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.codes, (uint64_t)w.code_stride,
                      (uint64_t)w.rows_pad, (uint64_t)w.code_stride, kRowBytes, BN,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  Params p;
  p.M = x.rows;
  p.N = w.rows;
  p.nk = w.code_stride / kRowBytes;
  p.nt_m = x.rows_pad / BM;
  p.nblk_b = w.rows_pad / 128;
  const int64_t tiles = (int64_t)p.nt_m * ceil_div(w.rows, BN);
  if (tiles < 1 || tiles >= INT32_MAX) return cudaErrorInvalidValue;
  p.tiles = (int)tiles;
  p.sf_chunks = w.sf_chunks;
  p.sfa = x.scales;
  p.sfb = w.scales;
  p.gx = x.g;
  p.gw = w.g;
  p.y = y;
  p.status = status;
  p.wait_ns = wait_ns;
  p.skip_stage = skip_stage;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::min<int64_t>(tiles, sms);
  CUtensorMap my;
  const bool tma_y = (p.N & 3) == 0 && (reinterpret_cast<uintptr_t>(y) & 15u) == 0 &&
                     tc05::make_map(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, y, (uint64_t)p.N, (uint64_t)p.M,
                                    (uint64_t)p.N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (tma_y) {
    if ((e = ensure_smem_attr((const void*)k_nvfp4_gemm<true>, kSmemBytes)) != cudaSuccess) return e;
    k_nvfp4_gemm<true><<<grid, kThreads, kSmemBytes, stream>>>(ma, mb, my, p);
  } else {
    if ((e = ensure_smem_attr((const void*)k_nvfp4_gemm<false>, kSmemBytes)) != cudaSuccess) return e;
    k_nvfp4_gemm<false><<<grid, kThreads, kSmemBytes, stream>>>(ma, mb, ma, p);
  }
  return cudaGetLastError();
}

}  // namespace sq
