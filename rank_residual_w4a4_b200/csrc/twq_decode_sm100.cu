// Decode-shape kernel (b <= 16 tokens) of the dual-component W4A4 + low-rank
// layer for sm_100a (TwinQuant, "Learnable Subspace Decomposition for 4-Bit
// LLM Quantization", §4.3 and Fig. 4; same arithmetic as twq_gemm_sm100.cu).
//
// With a handful of tokens the layer is a stream of the packed weights, so the
// kernel is laid out for HBM rather than for the tensor cores:
//   * swap-AB: the 128 output columns of a tile are the MMA's M side, the
//     tokens (padded to 16) its N side;
//   * split K: a cluster of KS CTAs shares one column tile; CTA k of the cluster
//     reduces over its own m/KS slice of the groups, so 4 x (n/128) CTAs stream
//     the weights at once;
//   * R and L1 codes: every group tile of the CTA is requested by TMA at once
//     (64-byte swizzle; R tiles by warp 0, L1 tiles by warp 2, in parallel);
//     warps unpack them in registers and write the int8 A operand straight into
//     tensor memory (tcgen05.st), so shared memory only carries the packed bytes
//     once;
//   * stage 1 gives each CTA a partial H (its groups) for all r; the partials
//     are pushed over distributed shared memory to the CTA that owns each
//     16-column unit of r, which sums them in a fixed order, rounds to BF16 and
//     runs its unit's share of stage 2 (H kept on chip, never in HBM);
//   * Y partials (residual over the CTA's groups + stage 2 over its r units)
//     are pushed to the CTA that owns each column slice, summed in a fixed
//     order, rounded to BF16 and stored once.
// Variants: the activation quantizer inside the kernel (BF16 X in, kQ), and
// W4A8 (int8 activation codes, q_max = 127, kA8). The kernel signals programmatic
// launch completion at entry; every role passes griddepcontrol.wait before it
// depends on X, which the preceding kernel may produce.
// Cross-CTA data moves only as st.async pushes into the receiving CTA's shared
// memory, each completing bytes on the receiver's mbarrier (which registered
// the exact byte count it expects before the cluster rendezvous). A CTA never
// reads a peer's shared memory, and every write into it has landed once its
// bounded wait completes, so no CTA exits while a peer may still write into it.
#include <atomic>
#include <mutex>
#include <cuda_bf16.h>

#include "sm100_ptx.cuh"
#include "twq_eq1.cuh"
#include "twq_internal.h"

namespace twq {

__device__ int g_decode_status;


namespace {

constexpr int kThreads = 640;        // 20 warps
constexpr int kNT = 16;               // token tile: N of every MMA
constexpr int kMaxGroups = 8;         // groups of 128 per CTA
constexpr int kRing = 4;              // tensor-memory ring depth (operands and accumulators)
constexpr int kTmemCols = 512;
constexpr int kColL1 = 0;             // kRing x 32: int8 L1 operand tiles
constexpr int kColR = 128;            // kRing x 32: int8 R operand tiles
constexpr int kColDh = 256;           // kMaxGroups x 16: stage-1 accumulators
constexpr int kColDres = 384;         // kMaxGroups x 16: residual accumulators
constexpr int kColDlr = 0;            // 16: stage-2 accumulator (L1 ring, free after stage 1)
constexpr uint64_t kWaitLimitNs = 2000000000ull;

enum DecodeSite : int {
  kDSiteX = 21, kDSiteR = 22, kDSiteL1 = 23, kDSiteAl = 24, kDSiteH = 25, kDSiteRes = 26,
  kDSiteAr = 27, kDSiteHReady = 28, kDSiteHb = 29, kDSiteL2 = 30, kDSiteLr = 31,
  kDSiteYReady = 32, kDSiteFinal = 33, kDSiteHq = 34, kDSiteHmax = 35,
};

template <int kMode>
struct DTraits {
  static constexpr bool res = kMode == kModeFused || kMode == kModeW4A4;
  static constexpr bool lr = kMode == kModeFused || kMode == kModeLowRank;
};

struct DecodeArgs {
  const float* sx;
  const float* sr;
  const float* sl1;
  uint16_t* y;
  int64_t b;
  int m, n, r, G;
  const uint8_t* l2q;  // INT4 stage 2: 4-bit L2 codes, n x r/2 (column j contiguous along r)
  const float* sl2q;   // INT4 stage 2: their scales, (r/128) x n
};

struct DLayout {
  static constexpr int kOffR = 0;                              // kMaxGroups x 8 KB (SW64)
  static constexpr int kOffL1 = kOffR + kMaxGroups * 8192;     // kMaxGroups x 8 KB (SW64)
  static constexpr int kOffXu = kOffL1 + kMaxGroups * 8192;    // kMaxGroups x 2 KB (SW128)
  static constexpr int kOffL2 = kOffXu + kMaxGroups * 2048;    // 16 KB (SW128)
  static constexpr int kOffHb = kOffL2 + 16384;                // 2 KB (SW128)
  static constexpr int kOffXp = kOffHb + 2048;                 // kMaxGroups x 1 KB codes, or
                                                               // kMaxGroups x 4 KB BF16 X
  static constexpr int kOffSx = kOffXp + kMaxGroups * 4096;    // [group][token] fp32
  static constexpr int kOffHred = kOffSx + kMaxGroups * kNT * 4;
  static constexpr int kHredBytes = 128 * kNT * 4;             // [src][c][t], KS * slice <= 128
  static constexpr int kOffYred = kOffHred + kHredBytes;
  static constexpr int kYredBytes = 128 * kNT * 4;             // [src][j][t], KS * cols = 128
  // INT4 stage 2: per-token maxima of |bf16(H)| from every CTA, s_H, this CTA's maxima
  static constexpr int kOffHmx = kOffYred + kYredBytes;        // [src][token] fp32
  static constexpr int kOffShq = kOffHmx + 8 * kNT * 4;         // [token] fp32
  static constexpr int kOffHloc = kOffShq + kNT * 4;            // [token] fp32 bits (atomicMax)
  static constexpr int kOffBar = kOffHloc + kNT * 4;
  static constexpr int kNumBars = 64;
  static constexpr int kBytes = kOffBar + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(DLayout::kAlloc <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ void d_fail(int site) { atomicCAS(&g_decode_status, 0, site); }

template <bool kCluster>
__device__ __noinline__ bool d_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int site) {
  auto probe = [&]() {
    return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (probe()) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      d_fail(site);
      *abort_flag = 1;
      return false;
    }
  }
}

// Bounded wait for `parity` on `bar`: one inline probe (the common case on the
// issuing threads, where the phase has often completed already), then the
// bounded loop. Gives up after kWaitLimitNs or once the CTA's abort flag is set.
template <bool kCluster>
__device__ __forceinline__ bool d_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                       int site) {
  if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  return d_wait_slow<kCluster>(bar, parity, abort_flag, site);
}

__device__ __forceinline__ uint8_t* d_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t d_sw128(int row, int c) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4));
}

// 8 packed bytes (16 codes) -> 16 int8 bytes holding 16*q; even-index codes first.
__device__ __forceinline__ void unpack8(uint32_t lo, uint32_t hi, uint32_t* o) {
  o[0] = (lo << 4) & 0xF0F0F0F0u;
  o[1] = lo & 0xF0F0F0F0u;
  o[2] = (hi << 4) & 0xF0F0F0F0u;
  o[3] = hi & 0xF0F0F0F0u;
}

// Row j of a TMA tile of 64-byte rows in the 64-byte swizzle -> 32 words of int8
// codes (16*q), stored into tensor-memory lane j, 32 columns from `col`.
__device__ __forceinline__ void tile_row_to_tmem(const uint8_t* tile, int j, uint32_t taddr) {
  const uint8_t* row = tile + j * 64;
  const int sw = (j >> 1) & 3;
  uint32_t v[32];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + ((c ^ sw) << 4));
    unpack8(w.x, w.y, &v[c * 8]);
    unpack8(w.z, w.w, &v[c * 8 + 4]);
  }
  tmem_st32(taddr, v);
}

// Eq. (1) quantizer fused into the prologue. The CTA's BF16 slice of X sits in
// shared memory as two TMA boxes per group (64 elements x 16 tokens each, rows
// of 128 bytes; tokens >= b read as zero). Four lanes take one (token, group)
// pair: lane l of the four covers the 16-element chunks l and l + 4 (elements
// [16 l, 16 l + 16) of each box). Quantizing lane `qi` of 320 (warps 2-3 and
// 12-19) handles the pairs qi / 4 + 80 k, so the 128 pairs of eight groups take
// two passes. Codes go to the 128-byte-swizzle B tiles as 16*q in the in-chunk
// order of unpack8, scales to sxs, with the arithmetic of twq_quantize_act, so
// the codes are identical (the group maximum is exact in any order).
constexpr int kQPairsPerPass = 80;  // 10 warps x 8 pairs


// 16 int8 codes (q_max = 127) in the same in-chunk order as pack_codes16.
__device__ __forceinline__ uint4 pack_codes16_a8(const uint32_t (&c)[16]) {
  uint4 o;
  o.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
  o.y = c[8] | (c[9] << 8) | (c[10] << 16) | (c[11] << 24);
  o.z = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
  o.w = c[12] | (c[13] << 8) | (c[14] << 16) | (c[15] << 24);
  return o;
}

// kA8: the W4A8 activations (q_max = 127): one int8 code q per byte, the same
// in-chunk order; else 16*q from a 4-bit code.
template <bool kA8>
__device__ __forceinline__ void quantize_slice(const uint8_t* xs, int ng, uint8_t* xu, float* sxs,
                                               uint64_t* xready, int qi, int lane) {
  const int l = lane & 3;
  const int pairs = kNT * ng;
  const int passes = (pairs + kQPairsPerPass - 1) / kQPairsPerPass;  // uniform over the warp
#pragma unroll 1
  for (int it = 0; it < passes; ++it) {
    const int p = (qi >> 2) + it * kQPairsPerPass;
    const bool pv = p < pairs;
    const int gi = pv ? p / kNT : 0, t = pv ? p % kNT : 0;
    const uint8_t* src = xs + gi * 4096 + t * 128 + l * 32;
    // f[h][0..7]: even elements 0, 2, .., 14 of chunk l + 4h; f[h][8..15]: odd elements
    float f[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 r0 = *reinterpret_cast<const uint4*>(src + h * 2048);
      const uint4 r1 = *reinterpret_cast<const uint4*>(src + h * 2048 + 16);
      const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        f[h][i] = __uint_as_float(w[i] << 16);
        f[h][8 + i] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
    float m4[4];  // absmax as a tree, for instruction-level parallelism
#pragma unroll
    for (int i = 0; i < 4; ++i)
      m4[i] = fmaxf(fmaxf(fmaxf(fabsf(f[0][i]), fabsf(f[0][i + 4])),
                          fmaxf(fabsf(f[0][i + 8]), fabsf(f[0][i + 12]))),
                    fmaxf(fmaxf(fabsf(f[1][i]), fabsf(f[1][i + 4])),
                          fmaxf(fabsf(f[1][i + 8]), fabsf(f[1][i + 12]))));
    float a = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
#pragma unroll
    for (int off = 2; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
    constexpr int kQmax = kA8 ? 127 : 7;
    const Eq1Scale ks = eq1_scale<kQmax>(a);
    uint4 o0 = make_uint4(0, 0, 0, 0), o1 = make_uint4(0, 0, 0, 0);
    if (ks.s != 0.0f) {
      uint32_t nb[16];
      eq1_codes<kQmax>(f[0], ks, nb);
      o0 = kA8 ? pack_codes16_a8(nb) : pack_codes16(nb);
      eq1_codes<kQmax>(f[1], ks, nb);
      o1 = kA8 ? pack_codes16_a8(nb) : pack_codes16(nb);
    }
    if (pv) {
      *reinterpret_cast<uint4*>(xu + gi * 2048 + d_sw128(t, l)) = o0;
      *reinterpret_cast<uint4*>(xu + gi * 2048 + d_sw128(t, l + 4)) = o1;
      if (l == 0) sxs[gi * kNT + t] = ks.s;
    }
    // Groups whose last pair falls in this pass are complete once every warp
    // has passed here: each warp arrives once on each of them.
    const int g_lo = it * kQPairsPerPass / kNT;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      for (int g = g_lo; g < ng; ++g) {
        const int done_pass = (g * kNT + kNT - 1) / kQPairsPerPass;
        if (done_pass == it) mbar_arrive(&xready[g]);
        if (done_pass > it) break;
      }
    }
  }
}

// Range of 16-column units of r owned by cluster rank k.
__device__ __forceinline__ void unit_range(int U, int KS, int k, int& u0, int& u1) {
  u0 = k * U / KS;
  u1 = (k + 1) * U / KS;
}

// kA8: W4A8, the activation codes are int8 (q_max = 127), one per byte.
// kS2Q: the INT4 stage 2 (H requantized on chip, 4-bit L2 codes), r = 128.
template <int kMode, int KS, bool kQ, bool kA8, bool kS2Q>
__global__ void __launch_bounds__(kThreads, 1)
    twq_decode_kernel(const __grid_constant__ CUtensorMap tm_rq,
                      const __grid_constant__ CUtensorMap tm_l1q,
                      const __grid_constant__ CUtensorMap tm_xq,
                      const __grid_constant__ CUtensorMap tm_l2t, const DecodeArgs args) {
  using L = DLayout;
  using T = DTraits<kMode>;
  // The weight operand holds 16*q (4-bit codes); X holds 16*q (W4A4) or q (W4A8):
  // an accumulator is 2^8 (2^4) times the group's integer dot product.
  constexpr float kDq = kA8 ? 0.0625f : 0.00390625f;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort;
  uint8_t* smem = d_align1024(smem_raw);
  uint8_t* rtiles = smem + L::kOffR;
  uint8_t* ltiles = smem + L::kOffL1;
  uint8_t* xu = smem + L::kOffXu;
  uint8_t* l2s = smem + L::kOffL2;
  uint8_t* hbs = smem + L::kOffHb;
  uint8_t* xp = smem + L::kOffXp;
  float* sxs = reinterpret_cast<float*>(smem + L::kOffSx);
  float* hred = reinterpret_cast<float*>(smem + L::kOffHred);
  float* yred = reinterpret_cast<float*>(smem + L::kOffYred);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* rfull = bars;                     // [kMaxGroups] TMA of R tiles
  uint64_t* lfull = rfull + kMaxGroups;       // [kMaxGroups] TMA of L1 tiles
  uint64_t* al_full = lfull + kMaxGroups;     // [kRing] L1 operand slot written
  // A ring slot is free again once the MMAs of the group that used it have completed,
  // which is what that group's accumulator barrier (h_full / res_full) records: one
  // tcgen05.commit per group serves both the drain and the next unpack into the slot.
  uint64_t* ar_full = al_full + kRing;        // [kRing] R operand slot written
  uint64_t* h_full = ar_full + kRing;         // [kMaxGroups] stage-1 accumulator ready
  uint64_t* res_full = h_full + kMaxGroups;   // [kMaxGroups] residual accumulator ready
  uint64_t* xfull = res_full + kMaxGroups;
  uint64_t* xready = xfull + 1;               // [kMaxGroups] group's X codes and scales ready
  uint64_t* l2full = xready + kMaxGroups;
  uint64_t* hb_ready = l2full + 1;
  uint64_t* lr_full = hb_ready + 1;
  uint64_t* h_ready = lr_full + 1;
  uint64_t* y_ready = h_ready + 1;
  uint64_t* mma_done = y_ready + 1;           // [2]
  uint64_t* hmax_ready = mma_done + 2;        // INT4 stage 2: every CTA's per-token maxima
  uint64_t* hq4 = mma_done + 3;               // INT4 stage 2: the 4 H-owner warps' maxima
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 4);
  float* hmx = reinterpret_cast<float*>(smem + L::kOffHmx);
  float* shq = reinterpret_cast<float*>(smem + L::kOffShq);
  int* hloc = reinterpret_cast<int*>(smem + L::kOffHloc);
  volatile int* abort_flag = &s_abort;

  // The next kernel on the stream may be scheduled now: its prologue and weight
  // loads overlap this grid, and it reads this grid's output only after its
  // griddepcontrol.wait, which waits for this grid to complete.
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ks = static_cast<int>(cluster_rank());
  const int n0 = blockIdx.y * 128;
  const int G = args.G;
  const int g0 = ks * G / KS;
  const int ng = (ks + 1) * G / KS - g0;
  const int U = args.r / 16;
  int u0 = 0, u1 = 0;
  if (T::lr) unit_range(U, KS, ks, u0, u1);
  const int my_units = u1 - u0;
  constexpr int kColsPerOwner = 128 / KS;
  constexpr int kHSlice = 128 / KS;  // r <= 128 here: at most 128/KS columns of r per CTA

  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tm_rq);
    tma_prefetch_desc(&tm_l1q);
    tma_prefetch_desc(&tm_xq);
    tma_prefetch_desc(&tm_l2t);
  }
  if (warp == 0) {
    // barrier init spread over the warp: lane i owns group i's copy barriers
    if (lane < kMaxGroups) {
      mbar_init(&xready[lane], kQ ? 10 : 2);
      mbar_init(&rfull[lane], 1);
      mbar_init(&h_full[lane], 1);
      mbar_init(&res_full[lane], 1);
    }
    if (lane < kRing) {
      mbar_init(&al_full[lane], 4);
      mbar_init(&ar_full[lane], 4);
    }
    if (lane == 31) {
      mbar_init(xfull, 1);
      mbar_init(l2full, 1);
      mbar_init(hb_ready, 4);
      mbar_init(lr_full, 1);
      // Exchange barriers complete on bytes: this CTA expects every peer's partials
      // for the r units and the column slice it owns (registered before the
      // cluster rendezvous, so before any peer can send).
      mbar_init(h_ready, 1);
      mbar_init(y_ready, 1);
      mbar_arrive_expect_tx(h_ready, KS * my_units * 16 * kNT * 4);
      mbar_arrive_expect_tx(y_ready, KS * kColsPerOwner * kNT * 4);
      mbar_init(mma_done, 1);
      mbar_init(mma_done + 1, 1);
      if (kS2Q) {  // every CTA sends its 16 per-token maxima to every CTA of the cluster
        mbar_init(hmax_ready, 1);
        mbar_arrive_expect_tx(hmax_ready, KS * kNT * 4);
        mbar_init(hq4, 4);
      }
      s_abort = 0;
    }
    if (kS2Q) {
      if (lane < kNT) hloc[lane] = 0;
      // the stage-2 B tile (H's codes) is zero beyond the CTA's slice of r (K padding)
      for (int e = lane; e < 2048 / 16; e += 32)
        reinterpret_cast<uint4*>(hbs)[e] = make_uint4(0, 0, 0, 0);
      // the MMAs read this tile through the async proxy: order the generic-proxy
      // zero-fill before them (the CTA barrier below then publishes it)
      fence_proxy_async_smem();
    }
    fence_barrier_init();
    __syncwarp();
    // Every copy of this CTA is requested before the cluster rendezvous (TMA writes
    // only this CTA's shared memory and completes on its own barriers): lane gi
    // issues group gi's tiles.
    if (lane < ng) {
      const int gi = lane;
      if (T::res) {
        mbar_arrive_expect_tx(&rfull[gi], 8192);
        tma_load_2d(rtiles + gi * 8192, &tm_rq, &rfull[gi], (g0 + gi) * 64, n0);
      }
    }
    if (lane == 31) {
      if (T::lr && my_units > 0 && !kS2Q) {
        mbar_arrive_expect_tx(l2full, 16384);
        tma_load_2d(l2s, &tm_l2t, l2full, u0 * 16, n0);
      }
    }
  }
  if (warp == 2) {
    // The L1 tiles are requested by warp 2 (idle here), in parallel with warp 0's R tiles:
    // a warp issues its lanes' TMA requests one after another.
    if (lane < kMaxGroups) mbar_init(&lfull[lane], 1);
    fence_barrier_init();
    __syncwarp();
    if (T::lr && lane < ng) {
      mbar_arrive_expect_tx(&lfull[lane], 8192);
      tma_load_2d(ltiles + lane * 8192, &tm_l1q, &lfull[lane], (g0 + lane) * 64, 0);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // Cluster rendezvous, split: every thread arrives here, after this CTA's barriers
  // are initialized; only the exchange warps (12-19), the ones that store into peers'
  // shared memory, wait for the peers' arrivals, just before their first push. The
  // arrive is relaxed: the initializations were published by fence.mbarrier_init
  // (release, cluster scope) in warps 0 and 2, and peers only write into this CTA.
  cluster_arrive_relaxed();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // Everything above overlaps the preceding kernel on the stream (programmatic
  // serialization). The activations may come from that kernel, so they are read
  // only after griddepcontrol.wait; so that no bounded wait below counts the
  // preceding kernel's run time, every role passes griddepcontrol.wait itself
  // before its first wait that depends on X.
  if (warp == 2 && lane == 0) {
    pdl_wait();
    if (kQ) {  // BF16 X: two boxes of 64 elements x 16 tokens per group
      mbar_arrive_expect_tx(xfull, ng * 4096);
      for (int gi = 0; gi < ng; ++gi) {
        tma_load_2d(xp + gi * 4096, &tm_xq, xfull, (g0 + gi) * 128, 0);
        tma_load_2d(xp + gi * 4096 + 2048, &tm_xq, xfull, (g0 + gi) * 128 + 64, 0);
      }
    } else {
      constexpr int kXBytes = kA8 ? 2048 : 1024;  // one group of 16 tokens: int8 or packed codes
      mbar_arrive_expect_tx(xfull, ng * kXBytes);
      for (int gi = 0; gi < ng; ++gi)
        tma_load_2d(xp + gi * kXBytes, &tm_xq, xfull, (g0 + gi) * (kXBytes / kNT), 0);
    }
  }
  __syncwarp();

  if (kQ && (warp == 2 || warp == 3 || warp >= 12)) {
    // ----- X quantize (warps 2-3 and 12-19; 12-19 then go on to their own roles)
    const int qi = (warp < 4 ? warp - 2 : warp - 10) * 32 + lane;
    pdl_wait();
    if (d_wait<false>(xfull, 0, abort_flag, kDSiteX)) quantize_slice<kA8>(xp, ng, xu, sxs, xready, qi, lane);
  }
  if (warp == 0) {
    // ------------------------------------ residual MMA issuer (lane 0 of warp 0)
    if (lane == 0) {
      pdl_wait();
      bool ok = true;
      const uint32_t xu0 = smem_u32(xu);
      const uint32_t idesc = idesc_i8(kNT);
      if (T::res) {
        for (int gi = 0; gi < ng && ok; ++gi) {
          const int slot = gi % kRing;
          const uint32_t ph = (gi / kRing) & 1;
          const uint64_t db = smem_desc_sw128(xu0 + gi * 2048);
          if (!(ok = d_wait<false>(&xready[gi], 0, abort_flag, kDSiteX))) break;
          if (!(ok = d_wait<false>(&ar_full[slot], ph, abort_flag, kDSiteAr))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8_tmem_a(tmem_base + kColDres + gi * 16, tmem_base + kColR + slot * 32 + k * 8,
                          db + 2 * k, idesc, k > 0);
          mma_commit(&res_full[gi]);
        }
      }
      mma_commit(mma_done + 1);
      // The CTA waits for its own copies and MMAs before it can finish.
      int never = 0;
      d_wait<false>(mma_done + 1, 0, &never, kDSiteFinal);
      d_wait<false>(xfull, 0, &never, kDSiteFinal);
      for (int gi = 0; gi < ng; ++gi) {
        if (T::lr) d_wait<false>(&lfull[gi], 0, &never, kDSiteFinal);
        if (T::res) d_wait<false>(&rfull[gi], 0, &never, kDSiteFinal);
      }
      if (T::lr && my_units > 0 && !kS2Q) d_wait<false>(l2full, 0, &never, kDSiteFinal);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      pdl_wait();
      bool ok = true;
      const uint32_t xu0 = smem_u32(xu);
      const uint32_t idesc = idesc_i8(kNT);
      for (int gi = 0; gi < ng && ok; ++gi) {
        const int slot = gi % kRing;
        const uint32_t ph = (gi / kRing) & 1;
        const uint64_t db = smem_desc_sw128(xu0 + gi * 2048);
        if (T::lr) {
          if (!(ok = d_wait<false>(&xready[gi], 0, abort_flag, kDSiteX))) break;
          if (!(ok = d_wait<false>(&al_full[slot], ph, abort_flag, kDSiteAl))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8_tmem_a(tmem_base + kColDh + gi * 16, tmem_base + kColL1 + slot * 32 + k * 8,
                          db + 2 * k, idesc, k > 0);
          mma_commit(&h_full[gi]);
        }
      }
      if (kS2Q && T::lr && my_units > 0 && ok) {
        // INT4 stage 2: A = this CTA's 4-bit L2 codes (128 columns x its slice of r, int8
        // 16q), B = the codes of H for the slice, K = the slice padded to 32
        ok = d_wait<true>(hb_ready, 0, abort_flag, kDSiteHb);
        if (ok) {
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(smem_u32(l2s));
          const uint64_t db = smem_desc_sw128(smem_u32(hbs));
          for (int k = 0; k < (my_units + 1) / 2; ++k)
            mma_i8(tmem_base + kColDlr, da + 2 * k, db + 2 * k, idesc, k > 0);
          mma_commit(lr_full);
        }
      } else if (T::lr && my_units > 0 && ok) {
        ok = d_wait<true>(hb_ready, 0, abort_flag, kDSiteHb) &&
             d_wait<false>(l2full, 0, abort_flag, kDSiteL2);
        if (ok) {
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(smem_u32(l2s));
          const uint64_t db = smem_desc_sw128(smem_u32(hbs));
          for (int u = 0; u < my_units; ++u)
            mma_bf16(tmem_base + kColDlr, da + 2 * u, db + 2 * u, idesc_bf16(kNT), u > 0);
          mma_commit(lr_full);
        }
      }
      mma_commit(mma_done);
      int never = 0;
      d_wait<false>(mma_done, 0, &never, kDSiteFinal);
    }
  } else if (warp < 4) {
    // the quantizing variant did its X work above; warps 2-3 have no other role
    if constexpr (!kQ) {
      // ------------------------------------------------ X unpack (warps 2 and 3)
      const int tid = threadIdx.x - 64;
      pdl_wait();    // the scales, like the codes, may come from the preceding kernel
      float sxv[2];  // activation scales, loaded before the codes arrive
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int e = tid + 64 * i;
        const int gi = e / kNT, t = e % kNT;
        sxv[i] = (gi < ng && t < args.b) ? __ldg(args.sx + static_cast<int64_t>(t) * G + g0 + gi) : 0.0f;
      }
      if (d_wait<false>(xfull, 0, abort_flag, kDSiteX)) {
        for (int e = tid; e < ng * kNT * 8; e += 64) {
          const int gi = e / (kNT * 8);
          const int row = (e / 8) % kNT;
          const int c = e & 7;
          uint32_t o[4];
          if constexpr (kA8) {  // 16 int8 codes in element order -> the MMA's in-chunk order
            const uint4 w = *reinterpret_cast<const uint4*>(xp + gi * 2048 + row * 128 + c * 16);
            o[0] = __byte_perm(w.x, w.y, 0x6420);  // elements 0, 2, 4, 6
            o[1] = __byte_perm(w.x, w.y, 0x7531);  // 1, 3, 5, 7
            o[2] = __byte_perm(w.z, w.w, 0x6420);  // 8, 10, 12, 14
            o[3] = __byte_perm(w.z, w.w, 0x7531);  // 9, 11, 13, 15
          } else {
            const uint2 w = *reinterpret_cast<const uint2*>(xp + gi * 1024 + row * 64 + c * 8);
            unpack8(w.x, w.y, o);
          }
          *reinterpret_cast<uint4*>(xu + gi * 2048 + d_sw128(row, c)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) sxs[tid + 64 * i] = sxv[i];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
          for (int g = 0; g < ng; ++g) mbar_arrive(&xready[g]);
      }
    }
  } else if (warp < 12) {
    // -------- operand tiles -> tensor memory: L1 (warps 4-7) and R (warps 8-11)
    const bool is_l1 = warp < 8;
    const int q = warp & 3;
    const int j = q * 32 + lane;  // tensor-memory lane: r index for L1, column for R
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    if (is_l1 ? T::lr : T::res) {
      uint64_t* tfull = is_l1 ? lfull : rfull;
      uint64_t* sfull = is_l1 ? al_full : ar_full;
      uint64_t* done = is_l1 ? h_full : res_full;  // [gi]: the MMAs of group gi completed
      const uint8_t* tiles = is_l1 ? ltiles : rtiles;
      const int col0 = is_l1 ? kColL1 : kColR;
      for (int gi = 0; gi < ng; ++gi) {
        const int slot = gi % kRing;
        if (!d_wait<false>(&tfull[gi], 0, abort_flag, is_l1 ? kDSiteL1 : kDSiteR)) break;
        // the first kRing slots are free from the start; a later group takes the slot of
        // group gi - kRing once that group's MMAs (which wait for X) have completed
        if (gi >= kRing) {
          if (gi == kRing) pdl_wait();
          if (!d_wait<false>(&done[gi - kRing], 0, abort_flag, is_l1 ? kDSiteAl : kDSiteAr)) break;
        }
        tc_fence_after();
        tile_row_to_tmem(tiles + gi * 8192, j, tmem_base + lane_addr + col0 + slot * 32);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfull[slot]);
      }
    }
  } else if (warp < 16) {
    // --------------- stage-1 drain, H exchange, BF16 H for stage 2 (warps 12-15)
    cluster_wait_acquire();  // peers' barriers are initialized before the first push
    pdl_wait();
    // INT4 stage 2: thread tid holds the 4-bit L2 codes of output column n0 + tid for this
    // CTA's units of r (8 bytes, 16 codes, per unit), loaded early
    uint2 l2w[4] = {};
    if (kS2Q && T::lr)
      for (int u = 0; u < my_units && u < 4; ++u)
        l2w[u] = __ldg(reinterpret_cast<const uint2*>(
            args.l2q + static_cast<int64_t>(n0 + threadIdx.x - 384) * (args.r / 2) + (u0 + u) * 8));
    if (T::lr) {
      const int q = warp & 3;
      const int c = q * 32 + lane;  // index into r
      const bool c_ok = c < args.r;
      const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
      float sl1v[kMaxGroups];
#pragma unroll
      for (int gi = 0; gi < kMaxGroups; ++gi)
        sl1v[gi] = (gi < ng && c_ok) ? __ldg(args.sl1 + static_cast<int64_t>(g0 + gi) * args.r + c) : 0.0f;
      float acc[kNT];
#pragma unroll
      for (int t = 0; t < kNT; ++t) acc[t] = 0.0f;
      // every quantizing warp arrives on the last group's barrier after all its scale
      // writes, so one wait makes every group's sxs visible
      bool ok = ng == 0 || d_wait<false>(&xready[ng - 1], 0, abort_flag, kDSiteX);
#pragma unroll
      for (int gi = 0; gi < kMaxGroups; ++gi) {
        if (gi < ng && ok) {
          if (!(ok = d_wait<false>(&h_full[gi], 0, abort_flag, kDSiteH))) break;
          tc_fence_after();
          uint32_t v[16];
          tmem_ld16(tmem_base + lane_addr + kColDh + gi * 16, v);
          tmem_wait_ld();
          const float* sxg = sxs + gi * kNT;
#pragma unroll
          for (int t = 0; t < kNT; ++t)
            acc[t] = fmaf(static_cast<float>(static_cast<int32_t>(v[t])) * sl1v[gi], sxg[t], acc[t]);
        }
      }
      tc_fence_before();
      // push this CTA's partial H for row c to the owner of c's 16-column unit
      // (pushed even after a local failure, so the exchange stays complete)
      if (c_ok) {
        const int u = c / 16;
        int owner = 0, ou0 = 0;
        for (int k = 0; k < KS; ++k) {
          int a0, a1;
          unit_range(U, KS, k, a0, a1);
          if (u >= a0 && u < a1) {
            owner = k;
            ou0 = a0;
          }
        }
        const int cl = c - ou0 * 16;
        const uint32_t dst = map_peer(smem_u32(hred + (ks * kHSlice + cl) * kNT), owner);
        const uint32_t rbar = map_peer(smem_u32(h_ready), owner);
#pragma unroll
        for (int t = 0; t < kNT; t += 4)
          st_async_peer_v4(dst + t * 4, acc[t] * kDq, acc[t + 1] * kDq, acc[t + 2] * kDq,
                           acc[t + 3] * kDq, rbar);
      }
      // An owner waits until every peer's bytes have landed (so none is still writing
      // into it when it exits); the wait ignores the abort flag for the same reason.
      int keep_waiting = 0;
      const bool got = my_units > 0 ? d_wait<true>(h_ready, 0, &keep_waiting, kDSiteHReady) : true;
      if constexpr (kS2Q) {
        // INT4 stage 2 (r = 128): Eq. (1) on bf16(H) per token over all of r. The CTAs
        // own slices of r, so each sends its per-token maxima to every CTA; all of them
        // then compute the same scale. Every step runs even after a local failure, so
        // the exchange stays complete and peers are not left waiting.
        const int tid = threadIdx.x - 384;
        const int slice = my_units * 16;  // <= 64
        const int t = tid & (kNT - 1);    // element e = tid + 128 i has token e % 16 = t
        float hv[8];
        float mx = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = tid + 128 * i;
          hv[i] = 0.0f;
          if (e < slice * kNT) {
            const int cl = e / kNT;
            float h = 0.0f;
            for (int k = 0; k < KS; ++k) h += hred[(k * kHSlice + cl) * kNT + t];
            hv[i] = __bfloat162float(__float2bfloat16_rn(h));  // H rounded to BF16 first
            mx = fmaxf(mx, fabsf(hv[i]));
          }
        }
        if (ok && got) atomicMax(hloc + t, __float_as_int(mx));  // non-negative: int order
        __syncwarp();
        if (lane == 0) mbar_arrive(hq4);
        int keep = 0;
        d_wait<false>(hq4, 0, &keep, kDSiteHq);
        if (tid < kNT)
          for (int k = 0; k < KS; ++k)
            st_async_peer_u32(map_peer(smem_u32(hmx + ks * kNT + tid), k),
                              static_cast<uint32_t>(hloc[tid]), map_peer(smem_u32(hmax_ready), k));
        const bool gotm = d_wait<true>(hmax_ready, 0, &keep, kDSiteHmax);
        float a = 0.0f;
        for (int k = 0; k < KS; ++k) a = fmaxf(a, hmx[k * kNT + t]);
        const Eq1Scale sh = eq1_scale<7>(a);
        if (tid < kNT) shq[tid] = sh.s;
        // codes of this thread's elements into the B tile (16 rows, SW128), as 16*q bytes in
        // the 4-bit operand order: even elements of each 16-element chunk first
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = tid + 128 * i;
          if (e < slice * kNT) {
            const int cl = e / kNT, w = cl & 15;
            uint32_t code = 0;
            if (sh.s != 0.0f) {
              const float f1[1] = {hv[i]};
              uint32_t nb[1];
              eq1_nibbles(f1, sh, nb);
              code = nb[0] << 4;
            }
            const int pos = (w & 8) + ((w & 1) ? 4 : 0) + ((w & 7) >> 1);
            hbs[d_sw128(t, cl >> 4) + pos] = static_cast<uint8_t>(code);
          }
        }
        // the A tile: 128 output columns x the slice of r, int8 16q (K padded to 32)
        {
          const int j = tid;
          for (int u = 0; u < 4; ++u) {
            if (u < ((my_units + 1) / 2) * 2) {
              uint32_t o[4] = {0, 0, 0, 0};
              if (u < my_units) unpack8(l2w[u].x, l2w[u].y, o);
              *reinterpret_cast<uint4*>(l2s + d_sw128(j, u)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
        (void)gotm;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(hb_ready);
      } else if (ok && got && my_units > 0) {
        const int tid = threadIdx.x - 384;
        const int slice = my_units * 16;
        for (int e = tid; e < slice * kNT; e += 128) {
          const int cl = e / kNT, t = e % kNT;
          float h = 0.0f;
          for (int k = 0; k < KS; ++k) h += hred[(k * kHSlice + cl) * kNT + t];
          *reinterpret_cast<__nv_bfloat16*>(hbs + d_sw128(t, cl >> 3) + (cl & 7) * 2) =
              __float2bfloat16_rn(h);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(hb_ready);
      }
    }
  } else {
    // ------------------------------- residual drain, Y exchange, store (warps 16-19)
    cluster_wait_acquire();  // peers' barriers are initialized before the first push
    pdl_wait();
    const int q = warp & 3;
    const int j = q * 32 + lane;  // column of the tile
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    float acc[kNT];
#pragma unroll
    for (int t = 0; t < kNT; ++t) acc[t] = 0.0f;
    bool ok = !T::res || ng == 0 || d_wait<false>(&xready[ng - 1], 0, abort_flag, kDSiteX);
    if (T::res) {
      float srv[kMaxGroups];
#pragma unroll
      for (int gi = 0; gi < kMaxGroups; ++gi)
        srv[gi] = gi < ng ? __ldg(args.sr + static_cast<int64_t>(g0 + gi) * args.n + n0 + j) : 0.0f;
#pragma unroll
      for (int gi = 0; gi < kMaxGroups; ++gi) {
        if (gi < ng && ok) {
          if (!(ok = d_wait<false>(&res_full[gi], 0, abort_flag, kDSiteRes))) break;
          tc_fence_after();
          uint32_t v[16];
          tmem_ld16(tmem_base + lane_addr + kColDres + gi * 16, v);
          tmem_wait_ld();
          const float* sxg = sxs + gi * kNT;
#pragma unroll
          for (int t = 0; t < kNT; ++t)
            acc[t] = fmaf(static_cast<float>(static_cast<int32_t>(v[t])) * srv[gi], sxg[t], acc[t]);
        }
      }
    }
    float part[kNT];
#pragma unroll
    for (int t = 0; t < kNT; ++t) part[t] = acc[t] * kDq;
    if (T::lr && my_units > 0 && ok) {
      // INT4 stage 2: s_V of column j for the group of r that holds this CTA's slice
      const float sv = kS2Q ? __ldg(args.sl2q + static_cast<int64_t>(u0 * 16 / 128) * args.n + n0 + j)
                            : 0.0f;
      if ((ok = d_wait<false>(lr_full, 0, abort_flag, kDSiteLr))) {
        tc_fence_after();
        uint32_t v[16];
        tmem_ld16(tmem_base + lane_addr + kColDlr, v);
        tmem_wait_ld();
        if constexpr (kS2Q) {
          // int32 = 256 x the codes' dot product over the slice; s_H from the H-owner warps,
          // complete once hb_ready completed (the MMA waited for it)
          ok = d_wait<false>(hb_ready, 0, abort_flag, kDSiteHb);
#pragma unroll
          for (int t = 0; t < kNT; ++t)
            part[t] += static_cast<float>(static_cast<int32_t>(v[t])) * sv * shq[t] * 0.00390625f;
        } else {
#pragma unroll
          for (int t = 0; t < kNT; ++t) part[t] += __uint_as_float(v[t]);
        }
      }
    }
    tc_fence_before();
    {  // push the partial of column j to the CTA that finalizes j's slice (always)
      const int owner = j / kColsPerOwner;
      const int jl = j % kColsPerOwner;
      const uint32_t dst = map_peer(smem_u32(yred + (ks * kColsPerOwner + jl) * kNT), owner);
      const uint32_t rbar = map_peer(smem_u32(y_ready), owner);
#pragma unroll
      for (int t = 0; t < kNT; t += 4)
        st_async_peer_v4(dst + t * 4, part[t], part[t + 1], part[t + 2], part[t + 3], rbar);
    }
    int keep_waiting = 0;  // not the abort flag: peers may still be writing into this CTA
    const bool got = d_wait<true>(y_ready, 0, &keep_waiting, kDSiteYReady);
    if (ok && got) {
      // A thread sums four consecutive tokens of one column (16-byte reads: a quarter
      // warp reads 128 contiguous bytes, so the loads are free of bank conflicts),
      // over the ranks in order.
      const int tid = threadIdx.x - 512;
      for (int e = tid; e < kColsPerOwner * (kNT / 4); e += 128) {
        const int tc = e & 3, jl = e >> 2;
        float yv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int k = 0; k < KS; ++k) {
          const float4 v = *reinterpret_cast<const float4*>(yred + (k * kColsPerOwner + jl) * kNT + tc * 4);
          yv[0] += v.x;
          yv[1] += v.y;
          yv[2] += v.z;
          yv[3] += v.w;
        }
        uint16_t* yc = args.y + n0 + ks * kColsPerOwner + jl;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = tc * 4 + i;
          if (t < args.b)
            yc[static_cast<int64_t>(t) * args.n] = __bfloat16_as_ushort(__float2bfloat16_rn(yv[i]));
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn d_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Encoded tensor maps by their parameters. A decode call is short, so the host
// cost of encoding its four maps matters; the weights' maps repeat on every call
// of a layer. A map only encodes an address and a shape, so a hit is exact.
struct MapKey {
  const void* base;
  uint64_t inner, outer, row_bytes;
  uint32_t box_inner, box_outer;
  int dt, sw;
  bool operator==(const MapKey& o) const {
    return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
           box_inner == o.box_inner && box_outer == o.box_outer && dt == o.dt && sw == o.sw;
  }
};
constexpr int kMapCacheSize = 256;  // direct-mapped
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool valid;
};
MapEntry g_map_cache[kMapCacheSize];
std::mutex g_map_mutex;

bool d_encode_raw(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle sw);

// Drops every cached map (twq_release_cache).
void clear_map_cache() {
  std::lock_guard<std::mutex> lock(g_map_mutex);
  for (MapEntry& e : g_map_cache) e.valid = false;
}

bool d_encode(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
              uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle sw) {
  const MapKey key{base, inner, outer, row_bytes, box_inner, box_outer, static_cast<int>(dt),
                   static_cast<int>(sw)};
  uint64_t h = reinterpret_cast<uintptr_t>(base) * 0x9E3779B97F4A7C15ull;
  h ^= (inner * 31 + outer) * 0xC2B2AE3D27D4EB4Full;
  h ^= (row_bytes + (uint64_t(box_inner) << 20) + (uint64_t(box_outer) << 40) + key.dt * 7 + key.sw);
  MapEntry& e = g_map_cache[(h >> 32) % kMapCacheSize];
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    if (e.valid && e.key == key) {
      *map = e.map;
      return true;
    }
  }
  if (!d_encode_raw(map, dt, base, inner, outer, row_bytes, box_inner, box_outer, sw)) return false;
  std::lock_guard<std::mutex> lock(g_map_mutex);
  e.key = key;
  e.map = *map;
  e.valid = true;
  return true;
}

bool d_encode_raw(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = d_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kMode, int KS, bool kQ, bool kA8, bool kS2Q = false>
cudaError_t launch_decode_mode(const GemmCall& c, cudaStream_t st) {
  const twq_weights* w = c.w;
  DecodeArgs a{};
  a.sx = c.sx;
  a.sr = w->sr;
  a.sl1 = w->sl1;
  a.y = static_cast<uint16_t*>(c.out);
  a.b = c.b;
  a.m = static_cast<int>(w->m);
  a.n = static_cast<int>(w->n);
  a.r = static_cast<int>(w->r);
  a.G = a.m / 128;
  CUtensorMap m_rq{}, m_l1q{}, m_xq{}, m_l2t{};
  const uint64_t kb = static_cast<uint64_t>(a.m / 2);
  bool ok = kQ ? d_encode(&m_xq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.x, a.m, c.b,
                          static_cast<uint64_t>(c.ldx) * 2, 64, kNT, CU_TENSOR_MAP_SWIZZLE_NONE)
           : kA8 ? d_encode(&m_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.xq, a.m, c.b, a.m, 128, kNT,
                            CU_TENSOR_MAP_SWIZZLE_NONE)
                 : d_encode(&m_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.xq, kb, c.b, kb, 64, kNT,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
  if (DTraits<kMode>::res)
    ok = ok && d_encode(&m_rq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->rq, kb, a.n, kb, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_64B);
  if (DTraits<kMode>::lr)
    ok = ok && d_encode(&m_l1q, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->l1q, kb, a.r, kb, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_64B);
  if (DTraits<kMode>::lr && !kS2Q)
    ok = ok && d_encode(&m_l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->l2t, a.r, a.n,
                        static_cast<uint64_t>(a.r) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (kS2Q) {
    a.l2q = c.l2q;
    a.sl2q = c.sl2q;
    ok = ok && c.l2q && c.sl2q;
  }
  if (!ok) return cudaErrorInvalidValue;
  auto kern = twq_decode_kernel<kMode, KS, kQ, kA8, kS2Q>;
  // The shared-memory opt-in is a driver call: once per instantiation and device.
  static std::atomic<uint64_t> smem_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (!bit || !(smem_set.load(std::memory_order_relaxed) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DLayout::kAlloc);
    if (e != cudaSuccess) return e;
    smem_set.fetch_or(bit);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(KS, a.n / 128, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = DLayout::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = KS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // Programmatic stream serialization: if the preceding kernel signals early
  // (twq_quantize_act does), this kernel's prologue and weight loads overlap it;
  // the activation reads wait for its completion (griddepcontrol.wait).
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, m_rq, m_l1q, m_xq, m_l2t, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool decode_eligible(const GemmCall& c) {
  const twq_weights* w = c.w;
  if (c.mode == kModeFusedS2Q) return !c.x && !c.a8 && c.b >= 1 && c.b <= kNT && w->r == 128 &&
                                      w->m / 128 <= 8 * kMaxGroups && w->n % 128 == 0;
  if (c.mode != kModeFused && c.mode != kModeW4A4 && c.mode != kModeLowRank) return false;
  if (c.a8 && c.mode == kModeLowRank) return false;
  if (c.b < 1 || c.b > kNT) return false;
  if (c.mode != kModeW4A4 && (w->r <= 0 || w->r > 128)) return false;
  const int64_t G = w->m / 128;
  return G <= 8 * kMaxGroups && w->n % 128 == 0;
}

cudaError_t launch_decode(const GemmCall& c, cudaStream_t st) {
  const int64_t G = c.w->m / 128;
  const bool ks8 = G > 4 * kMaxGroups;
  const bool q = c.x != nullptr;
#define TWQ_DECODE_CASE(MODE, A8)                                                          \
  if (q) return ks8 ? launch_decode_mode<MODE, 8, true, A8>(c, st)                        \
                    : launch_decode_mode<MODE, 4, true, A8>(c, st);                       \
  return ks8 ? launch_decode_mode<MODE, 8, false, A8>(c, st)                              \
             : launch_decode_mode<MODE, 4, false, A8>(c, st);
  if (c.mode == kModeFusedS2Q)  // the INT4 stage 2 (codes in, r = 128)
    return ks8 ? launch_decode_mode<kModeFused, 8, false, false, true>(c, st)
               : launch_decode_mode<kModeFused, 4, false, false, true>(c, st);
  if (c.a8) {  // W4A8: the full layer and the residual alone
    switch (c.mode) {
      case kModeFused: { TWQ_DECODE_CASE(kModeFused, true) }
      case kModeW4A4: { TWQ_DECODE_CASE(kModeW4A4, true) }
      default:
        return cudaErrorInvalidValue;
    }
  }
  switch (c.mode) {
    case kModeFused: { TWQ_DECODE_CASE(kModeFused, false) }
    case kModeW4A4: { TWQ_DECODE_CASE(kModeW4A4, false) }
    case kModeLowRank: { TWQ_DECODE_CASE(kModeLowRank, false) }
    default:
      return cudaErrorInvalidValue;
  }
#undef TWQ_DECODE_CASE
}

cudaError_t read_and_clear_decode_status(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_decode_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_decode_status, &zero, sizeof(int));
  *code = v;
  return e;
}

void release_decode_cache() { clear_map_cache(); }

}  // namespace twq
