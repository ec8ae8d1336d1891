// Prefill kernel of the dual-component W4A4 + low-rank linear layer on CTA pairs
// (TwinQuant, "Learnable Subspace Decomposition for 4-Bit LLM Quantization", §4.3
// "Dual-Component Kernel Design", Fig. 4; Eq. (2) applied group by group).
//
// A cluster of two CTAs shares every tensor-core MMA (tcgen05 cta_group::2): the
// pair computes a 256 x 256 output tile, each CTA holding 128 rows of X (the MMA's
// A) and 128 of the 256 output columns of the weights (its half of B), and each
// CTA's tensor memory holding its 128 rows of the tile's accumulator. Per pair tile:
//   * stage 1 (only when the row block changes): H = Q(X) Q(L1) over all m/128
//     groups (N = r); each group's exact int32 accumulator is scaled by
//     sx[i,g] * sl1[g,c] in fp32 and summed in registers; H -> BF16 into a
//     shared-memory operand tile that the pair's later tiles of the same row block
//     reuse (H never goes to HBM);
//   * residual: Y_res = sum_g sx[i,g] sr[g,j] (Q(X)_g Q(R)_g), same scheme (N = 256);
//   * stage 2: Y_lr = bf16(H) L2 with kind::f16 MMAs, fp32 accumulation in tensor memory;
//     or, in the INT4 stage-2 mode (§4.3 item 2), bf16(H) requantized on chip per token and
//     group of 128 along r (Eq. (1)), and Q_H Q(V) run as r/128 more int8 K groups of the
//     residual accumulation (scales s_H per token, s_V per column);
//   * one epilogue: Y = bf16(Y_res + Y_lr), a single store.
// The weight codes are unpacked to 16 q (two logic operations per four bytes). X
// arrives in one of two forms:
//   * kXB: one int8 code per element (4-bit codes stored in bytes, or the 8-bit codes
//     of W4A8): TMA puts the group straight into the MMA's operand slot, and the
//     accumulator is 16 x the group's integer dot product;
//   * packed nibbles: unpacked like the weights, and the accumulator is 256 x it.
// Either way the accumulator is exact and the final power-of-two scaling is exact.
//
// Warp roles (16 warps):
//   warp 0        TMA: X (kXB: one group per copy, even group steps; else packed,
//                 two groups per copy);
//   warp 1        tensor memory (both CTAs); in the even CTA, the MMA issuer;
//   warp 2        TMA: packed 4-bit R / L1 tiles (two groups per copy) and the
//                 per-group weight scales (four groups per copy); in the INT4 stage-2
//                 mode also the 4-bit V codes and their scales;
//   warp 3        kXB: TMA of X for the odd group steps (a thread issues a copy
//                 every few hundred cycles at best, so two share the X stream);
//   warps 4-7     unpack: 4-bit codes -> 16 q int8 in the MMA's 128-byte-swizzle
//                 K-major layout (even codes of each 8 first in both operands, or,
//                 with kXB, the weights in element order like the X codes);
//                 they also bring the BF16 L2^T chunks of stage 2 by TMA;
//   warps 8-15    drain: per-group tensor-memory loads of 16 columns, fp32 scaling
//                 and accumulation (packed f32x2 arithmetic), H -> BF16 (and, in the
//                 INT4 stage-2 mode, its requantization), epilogue.
// The drain warps hold 128 fp32 sums per thread: their warpgroups raise their
// register budget (setmaxnreg) and the others lower theirs.
//
// Each pair takes a contiguous run of tiles chosen on the host (partition_items) to
// balance tiles against stage-1 passes.
//
// Every wait is bounded; a wait that runs out records its site in a device status
// word, raises the CTA's abort flag, lets the CTA's copies in flight land, and the
// CTA leaves through the common teardown (MMAs complete, cluster barrier, tensor
// memory freed). No trap, no device assert.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "sm100_ptx.cuh"
#include "twq_hrequant.cuh"
#include "twq_internal.h"

namespace twq {

__device__ int g_pair_status;

namespace {

constexpr int kThreads = 512;
constexpr int kSS = 4;     // weight-scale slots, four K groups each (the weight producer
                           // loads them, so a deep ring keeps it ahead of the drain)
constexpr int kMaxR = 256;
constexpr int kMaxPairs = 128;  // runs in the launch's tile partition

// Wait sites of this kernel (recorded in g_pair_status).
enum PairSite : int {
  kPSiteXEmpty = 41, kPSiteBEmpty = 42, kPSiteScaleEmpty = 43, kPSiteUnpackFull = 44,
  kPSiteUnpackEmpty = 45, kPSiteL2 = 46, kPSiteMmaFull = 47, kPSiteMmaAcc = 48, kPSiteMmaH = 49,
  kPSiteDrainAcc = 50, kPSiteDrainScale = 51, kPSiteFinal = 52, kPSiteHq = 53,
};

// Shared memory. A packed slot holds two K groups: (unless kXB) X 128 rows x 128
// bytes, then the weights 128 rows x 128 bytes. An unpacked slot holds one K group of
// both operands as int8 (A 16 KB, then B 16 KB), or a stage-2 L2^T chunk in its B half.
template <bool kXB>
struct Layout {
  static constexpr int kPS = kXB ? 3 : 2;    // packed slots
  static constexpr int kUS = kXB ? 3 : 2;    // unpacked slots
  static constexpr int kPackX = kXB ? 0 : 16384;
  static constexpr int kPack = kPackX + 16384;
  static constexpr int kUHalf = 16384;
  static constexpr int kU = 2 * kUHalf;
  static constexpr int kOffPack = 0;
  static constexpr int kOffU = kOffPack + kPS * kPack;
  static constexpr int kOffH = kOffU + kUS * kU;
  static constexpr int kHBytes = 128 * kMaxR * 2;      // r/64 chunks of 128 x 64 BF16
  static constexpr int kOffScale = kOffH + kHBytes;
  static constexpr int kScaleSlot = 4 * 256 * 4;       // four groups of up to 256 columns
  static constexpr int kOffShq = kOffScale + kSS * kScaleSlot;  // INT4 stage 2: s_H, 128 x 2
  static constexpr int kOffBar = kOffShq + 128 * 2 * 4;
  static constexpr int kNumBars = 40;
  static constexpr int kBytes = kOffBar + kNumBars * 8 + 32;
  static constexpr int kAlloc = kBytes + 1024;         // room to align the base to 1 KB
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

struct PairArgs {
  const float* sx;
  uint16_t* y;
  int64_t b;
  int m, n, r, G;
  int col_tiles, num_items;  // pair tiles of 256 x 256
  int bounds[kMaxPairs + 1];  // pair p takes tiles [bounds[p], bounds[p + 1]) in row-block-major order
  unsigned long long wait_ns;
  int stall;  // self-test: no copy of X is issued, so every wait on X runs out
};

template <int kMode>
struct Traits {
  static constexpr bool s2q = kMode == kModeFusedS2Q;  // INT4 stage 2
  static constexpr bool res = kMode == kModeFused || kMode == kModeW4A4 || s2q;
  static constexpr bool h = kMode == kModeFused || kMode == kModeLowRank || s2q;
  static constexpr bool s2 = h && !s2q;                // BF16 stage 2 (kind::f16)
};

struct Ring {
  int idx = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++idx == n) {
      idx = 0;
      phase ^= 1u;
    }
  }
};

struct WaitCtx {
  volatile int* abort_flag;
  unsigned long long limit_ns;
};

__device__ __forceinline__ void record(int site) { atomicCAS(&g_pair_status, 0, site); }

// Bounded wait (barriers here complete on the peer CTA's arrivals and multicast
// commits as well as on local ones; acquire at CTA scope, matching the arrives).
__device__ __forceinline__ bool wait_slow(uint64_t* bar, uint32_t parity, const WaitCtx& w, int site) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort_flag) return false;
    if (global_timer_ns() - t0 > w.limit_ns) {
      record(site);
      *w.abort_flag = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_on(uint64_t* bar, uint32_t parity, const WaitCtx& w, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, w, site);
}

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Offset of logical 16-byte chunk c of row `row` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int row, int c) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4));
}

// The unpack of one K group, per thread: the 16-byte items e = t + 128 i (i < 4) of
// the 128 unpack threads, item e at row (e & 7) + 8 (e >> 5) and chunk (e >> 3) & 3
// of the group, so each group of 8 lanes reads and writes one chunk of 8 consecutive
// rows (distinct banks). Packed tiles: 128-byte rows of two groups with the 128-byte
// swizzle, group j in logical chunks 4j..4j+3 (chunk 4j + c = (c ^ (row & 7)) ^ 4j, so
// group 1 is group 0's offset XOR 64); unpacked tiles: 128-byte rows, chunks 2c and
// 2c + 1 (the second at the first's offset XOR 16).
struct UnpackPlan {
  uint32_t src[4];
  uint32_t dst[4];
  int row[4];
};
__device__ __forceinline__ UnpackPlan unpack_plan(int t) {
  UnpackPlan p;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = t + 128 * i;
    const int row = (e & 7) + 8 * (e >> 5);
    const int c = (e >> 3) & 3;
    p.row[i] = row;
    p.src[i] = sw128(row, c);
    p.dst[i] = sw128(row, 2 * c);
  }
  return p;
}
// kNatural: the weight codes in element order within each 16-byte chunk (to pair with
// int8 X codes, which TMA brings in element order), two byte permutes per 8 output
// bytes; else even elements first in each 8, the order both unpacked operands share.
template <bool kNatural>
__device__ __forceinline__ void unpack_group(const uint8_t* src, uint8_t* dst, int rows, int j,
                                             const UnpackPlan& p) {
  const uint32_t jx = static_cast<uint32_t>(j) << 6;
#pragma unroll  // fully: the plan's arrays stay in registers
  for (int i = 0; i < 4; ++i) {
    if (p.row[i] < rows) {
      const uint4 w = *reinterpret_cast<const uint4*>(src + (p.src[i] ^ jx));
      uint4 o0, o1;
      o0.x = (w.x << 4) & 0xF0F0F0F0u;  // 16 x elements 0, 2, 4, 6 of the word
      o0.y = w.x & 0xF0F0F0F0u;         // 16 x elements 1, 3, 5, 7
      o0.z = (w.y << 4) & 0xF0F0F0F0u;
      o0.w = w.y & 0xF0F0F0F0u;
      o1.x = (w.z << 4) & 0xF0F0F0F0u;
      o1.y = w.z & 0xF0F0F0F0u;
      o1.z = (w.w << 4) & 0xF0F0F0F0u;
      o1.w = w.w & 0xF0F0F0F0u;
      if constexpr (kNatural) {
        const uint4 e0 = o0, e1 = o1;
        o0 = make_uint4(__byte_perm(e0.x, e0.y, 0x5140), __byte_perm(e0.x, e0.y, 0x7362),
                        __byte_perm(e0.z, e0.w, 0x5140), __byte_perm(e0.z, e0.w, 0x7362));
        o1 = make_uint4(__byte_perm(e1.x, e1.y, 0x5140), __byte_perm(e1.x, e1.y, 0x7362),
                        __byte_perm(e1.z, e1.w, 0x5140), __byte_perm(e1.z, e1.w, 0x7362));
      }
      *reinterpret_cast<uint4*>(dst + p.dst[i]) = o0;
      *reinterpret_cast<uint4*>(dst + (p.dst[i] ^ 16u)) = o1;
    }
  }
}

// acc[i] += float(I[i]) * s[i] * sx for 16 columns whose codes are in v.
__device__ __forceinline__ void scale16(float* acc, const uint32_t (&v)[16], const float* s,
                                        uint64_t sxx) {
#pragma unroll
  for (int i = 0; i < 16; i += 4) {
    const float4 s4 = *reinterpret_cast<const float4*>(s + i);
    uint64_t a0 = f2_pack(acc[i], acc[i + 1]), a1 = f2_pack(acc[i + 2], acc[i + 3]);
    const uint64_t t0 = f2_mul(f2_pack(static_cast<float>(static_cast<int32_t>(v[i])),
                                       static_cast<float>(static_cast<int32_t>(v[i + 1]))),
                               f2_pack(s4.x, s4.y));
    const uint64_t t1 = f2_mul(f2_pack(static_cast<float>(static_cast<int32_t>(v[i + 2])),
                                       static_cast<float>(static_cast<int32_t>(v[i + 3]))),
                               f2_pack(s4.z, s4.w));
    a0 = f2_fma(t0, sxx, a0);
    a1 = f2_fma(t1, sxx, a1);
    f2_unpack(a0, acc[i], acc[i + 1]);
    f2_unpack(a1, acc[i + 2], acc[i + 3]);
  }
}

// A full 128-column drain of one group, 16 columns per tensor-memory load: a load
// returns in about 60 cycles, and the smaller register window leaves the scaling
// arithmetic more registers (the thread also holds 128 fp32 sums).
__device__ __forceinline__ void drain128(float (&acc)[128], uint32_t ta, const float* s,
                                         uint64_t sxx) {
#pragma unroll
  for (int c = 0; c < 128; c += 16) {
    uint32_t v[16];
    tmem_ld16(ta + c, v);
    tmem_wait_ld();
    scale16(acc + c, v, s + c, sxx);
  }
}

// The same for 8 columns (stage 1 with r/2 not a multiple of 128).
__device__ __forceinline__ void drain8(float* acc, uint32_t taddr, const float* s, uint64_t sxx) {
  uint32_t v[8];
  tmem_ld8(taddr, v);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    uint64_t a = f2_pack(acc[i], acc[i + 1]);
    const uint64_t t = f2_mul(f2_pack(static_cast<float>(static_cast<int32_t>(v[i])),
                                      static_cast<float>(static_cast<int32_t>(v[i + 1]))),
                              f2_pack(s[i], s[i + 1]));
    a = f2_fma(t, sxx, a);
    f2_unpack(a, acc[i], acc[i + 1]);
  }
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// A 4 x 4 transpose of 16-byte pieces within each aligned group of four lanes: piece s
// of lane i moves to piece i of lane s (two exchange rounds, lane distance 2 then 1).
// The epilogue uses it so that four lanes store one row's 64 contiguous bytes.
__device__ __forceinline__ void transpose4x4(uint32_t (&e)[4][4], int lane) {
#pragma unroll
  for (int m = 2; m >= 1; m >>= 1) {
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      if (s & m) continue;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t send = hi ? e[s][w] : e[s | m][w];
        const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, m);
        if (hi) e[s][w] = recv;
        else e[s | m][w] = recv;
      }
    }
  }
}

// The work of one pair tile, in the order every role walks it.
struct Item {
  int rb, ct;
  bool need_h;
};
__device__ __forceinline__ Item item_at(const PairArgs& a, int t, int t_begin, bool has_h) {
  Item it;
  it.rb = t / a.col_tiles;
  it.ct = t - it.rb * a.col_tiles;
  it.need_h = has_h && (t == t_begin || (t - 1) / a.col_tiles != it.rb);
  return it;
}

template <int kMode, bool kXB>
__global__ void __launch_bounds__(kThreads, 1)
    twq_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_r,
                    const __grid_constant__ CUtensorMap tm_l1, const __grid_constant__ CUtensorMap tm_l2,
                    const __grid_constant__ CUtensorMap tm_sr,
                    const __grid_constant__ CUtensorMap tm_sl1,
                    const __grid_constant__ CUtensorMap tm_sv, const PairArgs args) {
  using L = Layout<kXB>;
  using T = Traits<kMode>;
  constexpr int kPS = L::kPS;
  constexpr int kUS = L::kUS;
  // 2^-4 or 2^-8: the accumulators hold 16 (int8 X) or 256 (unpacked X) x the dot products
  constexpr float kDq = kXB ? 0.0625f : 0.00390625f;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort;
  uint8_t* smem = align1k(smem_raw);
  uint8_t* pack = smem + L::kOffPack;
  uint8_t* ustg = smem + L::kOffU;
  uint8_t* hb = smem + L::kOffH;
  float* scl = reinterpret_cast<float*>(smem + L::kOffScale);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* xfull = bars;                 // [kUS] kXB: X group landed in the unpacked slot
                                          // [kPS] else: X half of a packed slot landed
  uint64_t* bfull = xfull + 3;            // [kPS] weight half of a packed slot landed
  uint64_t* pempty = bfull + 3;           // [kPS] unpack warps are done with the slot
  uint64_t* ufull = pempty + 3;           // [kUS] (even CTA) both CTAs' unpacked slot is ready
  uint64_t* uempty = ufull + 3;           // [kUS] the pair's MMAs are done with the slot
  uint64_t* l2full = uempty + 3;          // [kUS] a stage-2 L2^T chunk landed in the slot
  uint64_t* afull = l2full + 3;           // [2] an accumulator buffer is complete
  uint64_t* aempty = afull + 2;           // [2] (even CTA) both CTAs drained the buffer
  uint64_t* sfull = aempty + 2;           // [kSS] weight scales landed
  uint64_t* sempty = sfull + kSS;         // [kSS] drain warps are done with them
  uint64_t* hready = sempty + kSS;        // (even CTA) both CTAs' BF16 H tiles are written
  uint64_t* mdone = hready + 1;           // every MMA of the pair has completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  uint64_t* hq = mdone + 2;               // INT4 stage 2: the 8 drain warps' H steps
  float* shq = reinterpret_cast<float*>(smem + L::kOffShq);  // INT4 stage 2: s_H [row][group]
  static_assert(!(kXB && T::s2q), "the INT4 stage 2 runs on packed codes");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int G = args.G;
  const int r = args.r;
  const int KC = T::s2 ? (r + 63) / 64 : 0;  // BF16 stage-2 chunks of 64 along r
  const int NQ = T::s2q ? r / 128 : 0;        // INT4 stage 2: groups of 128 along r
  const int slots = (G + 1) / 2;  // packed slots per pass over the K groups
  const WaitCtx wc{&s_abort, args.wait_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < 3; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&bfull[i], 1);
      mbar_init(&pempty[i], 4);
      mbar_init(&ufull[i], 8);  // 4 unpack warps of each CTA
      mbar_init(&uempty[i], 1);
      mbar_init(&l2full[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&afull[i], 1);
      mbar_init(&aempty[i], 16);  // 8 drain warps of each CTA
    }
    for (int i = 0; i < kSS; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sempty[i], 8);
    }
    mbar_init(hready, 16);
    mbar_init(mdone, 1);
    mbar_init(hq, 8);
    s_abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tm_x);
    if (T::res) {
      tma_prefetch_desc(&tm_r);
      tma_prefetch_desc(&tm_sr);
    }
    if (T::h) {
      tma_prefetch_desc(&tm_l1);
      tma_prefetch_desc(&tm_l2);
      tma_prefetch_desc(&tm_sl1);
    }
    if (T::s2q) tma_prefetch_desc(&tm_sv);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers exist and their tensor memory is allocated before any
  // remote arrive, multicast commit or MMA.
  cluster_sync_startup();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int pairs = static_cast<int>(gridDim.x) >> 1;
  const int t_begin = args.bounds[pair];
  const int t_end = args.bounds[pair + 1];
  (void)pairs;
  const int row_half = static_cast<int>(rank) * 128;  // this CTA's rows / columns in the pair tile

  if (warp < 8) {
  // Register budgets: warps 0-7 give registers up to the drain warpgroups (8-15),
  // which hold 128 fp32 sums per thread: 256 x 64 + 256 x 192 = 65536, the
  // 512 x 128 registers the CTA is launched with (ptxas: 128 per thread).
  warpgroup_regs_dec<64>();
  if (warp == 0 || (kXB && warp == 3)) {
    // ------------------------------------------------------------------ TMA: X
    if (lane == 0) {
      uint32_t pend = 0, pend_ph = 0;  // per slot: a copy was requested; its phase
      bool ok = !args.stall;
      if constexpr (kXB) {
        // one K group per copy, into the A half of the unpacked slot; warp 0 takes the
        // even group steps and warp 3 the odd ones. Each of the two waits for every
        // step's slot in ring order, its own or not (and the stage-2 steps, which bring
        // no X): a parity wait only tells phases apart one at a time, and a producer
        // that skipped steps could find a slot's barrier two phases behind and take
        // the slot while its last use is still pending.
        // xph: per unpacked slot, the phase of its next X copy (slots also serve
        // stage-2 steps, which bring no X, so this differs from the ring's phase)
        const int mine = warp == 0 ? 0 : 1;
        Ring u;
        int gstep = 0;
        uint32_t xph = 0;
        for (int t = t_begin; t < t_end && ok; ++t) {
          const Item it = item_at(args, t, t_begin, T::h);
          for (int pass = 0; pass < 2 && ok; ++pass) {
            if (pass == 0 ? !it.need_h : !T::res) continue;
            for (int g = 0; g < G; ++g, ++gstep) {
              if (!(ok = wait_on(&uempty[u.idx], u.phase ^ 1u, wc, kPSiteXEmpty))) break;
              if ((gstep & 1) == mine) {
                mbar_arrive_expect_tx(&xfull[u.idx], 16384);
                tma_load_2d(ustg + u.idx * L::kU, &tm_x, &xfull[u.idx], g * 128,
                            it.rb * 256 + row_half);
                pend |= 1u << u.idx;
                pend_ph = (pend_ph & ~(1u << u.idx)) | (((xph >> u.idx) & 1u) << u.idx);
              }
              xph ^= 1u << u.idx;
              u.next(kUS);
            }
          }
          if (T::h) {
            for (int kc = 0; kc < KC && ok; ++kc) {  // stage-2 steps: not X's, waited all the same
              ok = wait_on(&uempty[u.idx], u.phase ^ 1u, wc, kPSiteXEmpty);
              u.next(kUS);
            }
          }
        }
      } else {
        Ring p;
        for (int t = t_begin; t < t_end && ok; ++t) {
          const Item it = item_at(args, t, t_begin, T::h);
          for (int pass = 0; pass < 2 && ok; ++pass) {
            if (pass == 0 ? !it.need_h : !T::res) continue;
            for (int gp = 0; gp < slots; ++gp) {
              if (!(ok = wait_on(&pempty[p.idx], p.phase ^ 1u, wc, kPSiteXEmpty))) break;
              mbar_arrive_expect_tx(&xfull[p.idx], 16384);
              tma_load_2d(pack + p.idx * L::kPack, &tm_x, &xfull[p.idx], gp * 128,
                          it.rb * 256 + row_half);
              pend |= 1u << p.idx;
              pend_ph = (pend_ph & ~(1u << p.idx)) | (p.phase << p.idx);
              p.next(kPS);
            }
          }
          if (T::s2q && ok) {  // the V groups' packed slot brings no X: complete its barrier
            if (!(ok = wait_on(&pempty[p.idx], p.phase ^ 1u, wc, kPSiteXEmpty))) break;
            mbar_arrive(&xfull[p.idx]);
            p.next(kPS);
          }
        }
      }
      if (!ok) {
        // Leaving early: the copies already requested land before the CTA exits.
        int never = 0;
        const WaitCtx wf{&never, args.wait_ns};
        for (int i = 0; i < 3; ++i)
          if ((pend >> i) & 1u) wait_on(&xfull[i], (pend_ph >> i) & 1u, wf, kPSiteFinal);
      }
    }
  } else if (warp == 2) {
    // ---------------------------------------- TMA: weight tiles and weight scales
    if (lane == 0) {
      Ring p, q;
      uint32_t pend = 0, pend_ph = 0, spend = 0, spend_ph = 0;
      bool ok = true;
      const int brows_h = r / 2;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const Item it = item_at(args, t, t_begin, T::h);
        for (int pass = 0; pass < 2 && ok; ++pass) {
          const bool h_pass = pass == 0;
          if (h_pass ? !it.need_h : !T::res) continue;
          for (int gp = 0; gp < slots; ++gp) {
            if ((gp & 1) == 0) {  // scales of groups 2 gp .. 2 gp + 3
              if (!(ok = wait_on(&sempty[q.idx], q.phase ^ 1u, wc, kPSiteScaleEmpty))) break;
              const int cols = h_pass ? r : 256;
              mbar_arrive_expect_tx(&sfull[q.idx], cols * 4 * 4);
              tma_load_2d(scl + q.idx * (L::kScaleSlot / 4), h_pass ? &tm_sl1 : &tm_sr,
                          &sfull[q.idx], h_pass ? 0 : it.ct * 256, 2 * gp);
              spend |= 1u << q.idx;
              spend_ph = (spend_ph & ~(1u << q.idx)) | (q.phase << q.idx);
              q.next(kSS);
            }
            if (!(ok = wait_on(&pempty[p.idx], p.phase ^ 1u, wc, kPSiteBEmpty))) break;
            uint8_t* dst = pack + p.idx * L::kPack + L::kPackX;
            const int brows = h_pass ? brows_h : 128;
            mbar_arrive_expect_tx(&bfull[p.idx], brows * 128);
            if (h_pass)
              tma_load_2d(dst, &tm_l1, &bfull[p.idx], gp * 128, static_cast<int>(rank) * brows_h);
            else
              tma_load_2d(dst, &tm_r, &bfull[p.idx], gp * 128, it.ct * 256 + row_half);
            pend |= 1u << p.idx;
            pend_ph = (pend_ph & ~(1u << p.idx)) | (p.phase << p.idx);
            p.next(kPS);
          }
        }
        if (T::s2q && ok) {
          // INT4 stage 2: the V groups' scales s_V (rows beyond r/128 read as zeros) and
          // this CTA's 128 columns of the 4-bit V codes, both groups in one copy (the
          // half beyond r/2 bytes reads as zeros when r = 128)
          if (!(ok = wait_on(&sempty[q.idx], q.phase ^ 1u, wc, kPSiteScaleEmpty))) break;
          mbar_arrive_expect_tx(&sfull[q.idx], 256 * 4 * 4);
          tma_load_2d(scl + q.idx * (L::kScaleSlot / 4), &tm_sv, &sfull[q.idx], it.ct * 256, 0);
          spend |= 1u << q.idx;
          spend_ph = (spend_ph & ~(1u << q.idx)) | (q.phase << q.idx);
          q.next(kSS);
          if (!(ok = wait_on(&pempty[p.idx], p.phase ^ 1u, wc, kPSiteBEmpty))) break;
          mbar_arrive_expect_tx(&bfull[p.idx], 128 * 128);
          tma_load_2d(pack + p.idx * L::kPack + L::kPackX, &tm_l2, &bfull[p.idx], 0,
                      it.ct * 256 + row_half);
          pend |= 1u << p.idx;
          pend_ph = (pend_ph & ~(1u << p.idx)) | (p.phase << p.idx);
          p.next(kPS);
        }
      }
      if (!ok) {
        int never = 0;
        const WaitCtx wf{&never, args.wait_ns};
        for (int i = 0; i < kPS; ++i)
          if ((pend >> i) & 1u) wait_on(&bfull[i], (pend_ph >> i) & 1u, wf, kPSiteFinal);
        for (int i = 0; i < kSS; ++i)
          if ((spend >> i) & 1u) wait_on(&sfull[i], (spend_ph >> i) & 1u, wf, kPSiteFinal);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (leader && lane == 0) {
      Ring u, a;
      uint32_t h_phase = 0;
      bool ok = true;
      const uint32_t u0 = smem_u32(ustg);
      const uint32_t h0 = smem_u32(hb);
      for (int t = t_begin; t < t_end && ok; ++t) {
        const Item it = item_at(args, t, t_begin, T::h);
        for (int pass = 0; pass < 2 && ok; ++pass) {
          const bool h_pass = pass == 0;
          if (h_pass ? !it.need_h : !T::res) continue;
          const uint32_t idesc = idesc_i8_m256(h_pass ? r : 256);
          for (int g = 0; g < G; ++g) {
            if (!(ok = wait_on(&ufull[u.idx], u.phase, wc, kPSiteMmaFull))) break;
            if (!(ok = wait_on(&aempty[a.idx], a.phase ^ 1u, wc, kPSiteMmaAcc))) break;
            tc_fence_after();
            const uint32_t d = tmem + a.idx * 256;
            const uint64_t da = smem_desc_sw128(u0 + u.idx * L::kU);
            const uint64_t db = smem_desc_sw128(u0 + u.idx * L::kU + L::kUHalf);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_i8_pair(d, da + 2 * k, db + 2 * k, idesc, k > 0);
            mma_commit_pair(&uempty[u.idx]);
            mma_commit_pair(&afull[a.idx]);
            u.next(kUS);
            a.next(2);
          }
        }
        if (T::s2q && ok) {
          // INT4 stage 2: Q_H Q(V), A = this row block's requantized H of group g2 (16*q
          // codes over the group's first 16 KB of the H tile, in both CTAs)
          if (it.need_h) {
            if (!(ok = wait_on(hready, h_phase, wc, kPSiteMmaH))) break;
            h_phase ^= 1u;
          }
          const uint32_t idesc = idesc_i8_m256(256);
          for (int g2 = 0; g2 < NQ; ++g2) {
            if (!(ok = wait_on(&ufull[u.idx], u.phase, wc, kPSiteMmaFull))) break;
            if (!(ok = wait_on(&aempty[a.idx], a.phase ^ 1u, wc, kPSiteMmaAcc))) break;
            tc_fence_after();
            const uint32_t d = tmem + a.idx * 256;
            const uint64_t da = smem_desc_sw128(h0 + g2 * 32768);
            const uint64_t db = smem_desc_sw128(u0 + u.idx * L::kU + L::kUHalf);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_i8_pair(d, da + 2 * k, db + 2 * k, idesc, k > 0);
            mma_commit_pair(&uempty[u.idx]);
            mma_commit_pair(&afull[a.idx]);
            u.next(kUS);
            a.next(2);
          }
        }
        if (T::s2 && ok) {
          // stage 2: bf16(H) (this row block's, on chip in both CTAs) x L2^T chunks
          if (it.need_h) {
            if (!(ok = wait_on(hready, h_phase, wc, kPSiteMmaH))) break;
            h_phase ^= 1u;
          }
          if (!(ok = wait_on(&aempty[a.idx], a.phase ^ 1u, wc, kPSiteMmaAcc))) break;
          const uint32_t idesc = idesc_bf16_m256(256);
          const uint32_t d = tmem + a.idx * 256;
          for (int kc = 0; kc < KC; ++kc) {
            if (!(ok = wait_on(&ufull[u.idx], u.phase, wc, kPSiteMmaFull))) break;
            tc_fence_after();
            const uint64_t da = smem_desc_sw128(h0 + kc * 16384);
            const uint64_t db = smem_desc_sw128(u0 + u.idx * L::kU + L::kUHalf);
            const int ksteps = min(4, (r - kc * 64) / 16);
            for (int k = 0; k < ksteps; ++k)
              mma_bf16_pair(d, da + 2 * k, db + 2 * k, idesc, (kc | k) != 0);
            mma_commit_pair(&uempty[u.idx]);
            u.next(kUS);
          }
          if (!ok) break;
          mma_commit_pair(&afull[a.idx]);
          a.next(2);
        }
      }
      // Every MMA of the pair completes before either CTA frees its tensor memory.
      mma_commit_pair(mdone);
    }
    if (lane == 0) {
      int never = 0;
      const WaitCtx wf{&never, args.wait_ns};
      wait_on(mdone, 0, wf, kPSiteFinal);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ unpack
    const UnpackPlan plan = unpack_plan(threadIdx.x - 128);
    const uint32_t ufull_lead = map_peer(smem_u32(ufull), 0);
    Ring p, u;
    uint32_t l2_phase = 0;  // per unpacked slot: phase of its next L2^T chunk copy
    uint32_t xph = 0;       // per unpacked slot: phase of its next X copy (kXB)
    bool ok = true;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Item it = item_at(args, t, t_begin, T::h);
      for (int pass = 0; pass < 2 && ok; ++pass) {
        const bool h_pass = pass == 0;
        if (h_pass ? !it.need_h : !T::res) continue;
        const int brows = h_pass ? r / 2 : 128;
        for (int g = 0; g < G; ++g) {
          const int j = g & 1;
          if (j == 0) {
            if (!kXB) ok = __all_sync(~0u, wait_on(&xfull[p.idx], p.phase, wc, kPSiteUnpackFull));
            if (ok) ok = __all_sync(~0u, wait_on(&bfull[p.idx], p.phase, wc, kPSiteUnpackFull));
            if (!ok) break;
          }
          if (!(ok = __all_sync(~0u, wait_on(&uempty[u.idx], u.phase ^ 1u, wc, kPSiteUnpackEmpty))))
            break;
          const uint8_t* src = pack + p.idx * L::kPack;
          uint8_t* dst = ustg + u.idx * L::kU;
          if (!kXB) unpack_group<false>(src, dst, 128, j, plan);
          unpack_group<kXB>(src + L::kPackX, dst + L::kUHalf, brows, j, plan);
          fence_proxy_async_smem();
          if (kXB) {  // X arrives by TMA into the same slot: the MMA may start once it has
            ok = __all_sync(~0u, wait_on(&xfull[u.idx], (xph >> u.idx) & 1u, wc, kPSiteUnpackFull));
            xph ^= 1u << u.idx;
            if (!ok) break;
          }
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_cluster_n(ufull_lead + u.idx * 8, 1);
            if (j == 1 || g == G - 1) mbar_arrive(&pempty[p.idx]);
          }
          if (j == 1 || g == G - 1) p.next(kPS);
          u.next(kUS);
        }
      }
      if (T::s2q && ok) {
        // INT4 stage 2: the V groups, B only (A is the requantized H, already on chip)
        for (int g2 = 0; g2 < NQ; ++g2) {
          const int j = g2 & 1;
          if (j == 0) {
            ok = __all_sync(~0u, wait_on(&xfull[p.idx], p.phase, wc, kPSiteUnpackFull));
            if (ok) ok = __all_sync(~0u, wait_on(&bfull[p.idx], p.phase, wc, kPSiteUnpackFull));
            if (!ok) break;
          }
          if (!(ok = __all_sync(~0u, wait_on(&uempty[u.idx], u.phase ^ 1u, wc, kPSiteUnpackEmpty))))
            break;
          unpack_group<false>(pack + p.idx * L::kPack + L::kPackX, ustg + u.idx * L::kU + L::kUHalf,
                              128, j, plan);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_cluster_n(ufull_lead + u.idx * 8, 1);
            if (j == 1 || g2 == NQ - 1) mbar_arrive(&pempty[p.idx]);
          }
          if (j == 1 || g2 == NQ - 1) p.next(kPS);
          u.next(kUS);
        }
      }
      if (T::s2 && ok) {
        // stage 2: the L2^T chunks (this CTA's 128 columns x 64 of r, BF16, 128-byte
        // swizzle) go by TMA straight into the weight half of the unpacked slots
        for (int kc = 0; kc < KC; ++kc) {
          if (!(ok = __all_sync(~0u, wait_on(&uempty[u.idx], u.phase ^ 1u, wc, kPSiteUnpackEmpty))))
            break;
          if (warp == 4) {
            bool landed = true;
            if (lane == 0) {
              mbar_arrive_expect_tx(&l2full[u.idx], 16384);
              tma_load_2d(ustg + u.idx * L::kU + L::kUHalf, &tm_l2, &l2full[u.idx], kc * 64,
                          it.ct * 256 + row_half);
              // Wait for the copy even when the CTA is aborting: it has been issued and
              // must land before the CTA leaves.
              int never = 0;
              const WaitCtx wf{&never, args.wait_ns};
              landed = wait_on(&l2full[u.idx], (l2_phase >> u.idx) & 1u, wf, kPSiteL2);
              if (landed)  // for the CTA's 4 unpack warps
                mbar_arrive_cluster_n(ufull_lead + u.idx * 8, 4);
              else
                s_abort = 1;
            }
            l2_phase ^= 1u << u.idx;
            if (!(ok = __shfl_sync(~0u, landed ? 1 : 0, 0) != 0)) break;
          }
          u.next(kUS);
        }
      }
    }
  }
  } else {
    // ------------------------------------------------------------------- drain
    warpgroup_regs_inc<192>();
    const int dw = warp - 8;
    const int quarter = warp & 3;  // tensor-memory lane quarter this warp may access
    const int half = dw >> 2;      // which half of the tile's columns
    const int row_in = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t aempty_lead = map_peer(smem_u32(aempty), 0);
    const uint32_t hready_lead = map_peer(smem_u32(hready), 0);
    Ring a, q;
    bool ok = true;
    uint32_t hq_phase = 0;  // INT4 stage 2: the phase of the drain warps' barrier
    float acc[128];
    for (int t = t_begin; t < t_end && ok; ++t) {
      const Item it = item_at(args, t, t_begin, T::h);
      const int64_t grow = static_cast<int64_t>(it.rb) * 256 + row_half + row_in;
      const bool row_ok = grow < args.b;
      const float* sx_row = args.sx + (row_ok ? grow : 0) * G;
      for (int pass = 0; pass < 2 && ok; ++pass) {
        const bool h_pass = pass == 0;
        if (h_pass ? !it.need_h : !T::res) continue;
        const int ncols = h_pass ? r / 2 : 128;
        const int cstride = h_pass ? r : 256;  // floats per group in a scale slot
        const int c0 = half * ncols;
#pragma unroll
        for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
        float sxn = row_ok ? __ldg(sx_row) : 0.0f;
        for (int g = 0; g < G; ++g) {
          const float sxv = sxn;
          sxn = (row_ok && g + 1 < G) ? __ldg(sx_row + g + 1) : 0.0f;
          if ((g & 3) == 0)
            if (!(ok = __all_sync(~0u, wait_on(&sfull[q.idx], q.phase, wc, kPSiteDrainScale)))) break;
          if (!(ok = __all_sync(~0u, wait_on(&afull[a.idx], a.phase, wc, kPSiteDrainAcc)))) break;
          tc_fence_after();
          const uint64_t sxx = f2_pack(sxv, sxv);
          const uint32_t ta = tmem + lane_addr + a.idx * 256 + c0;
          const float* s = scl + q.idx * (L::kScaleSlot / 4) + (g & 3) * cstride + c0;
          if (ncols == 128) {
            drain128(acc, ta, s, sxx);
          } else {
#pragma unroll
            for (int c = 0; c < 128; c += 8)
              if (c < ncols) drain8(acc + c, ta + c, s + c, sxx);
          }
          tc_fence_before();
          __syncwarp();
          const bool slot_done = (g & 3) == 3 || g == G - 1;
          if (lane == 0) {
            mbar_arrive_cluster_n(aempty_lead + a.idx * 8, 1);
            if (slot_done) mbar_arrive(&sempty[q.idx]);
          }
          a.next(2);
          if (slot_done) q.next(kSS);
        }
        if (!ok) break;
        if (h_pass) {
          // H complete for this row block: kDq undoes the code scaling; BF16 into the
          // stage-2 operand tile (row row_in, columns c0 .. c0 + ncols).
#pragma unroll
          for (int j = 0; j < 128; j += 8) {
            if (j < ncols) {
              uint4 o;
              o.x = bf16x2(acc[j + 0] * kDq, acc[j + 1] * kDq);
              o.y = bf16x2(acc[j + 2] * kDq, acc[j + 3] * kDq);
              o.z = bf16x2(acc[j + 4] * kDq, acc[j + 5] * kDq);
              o.w = bf16x2(acc[j + 6] * kDq, acc[j + 7] * kDq);
              const int col = c0 + j;
              *reinterpret_cast<uint4*>(hb + (col >> 6) * 16384 + sw128(row_in, (col & 63) >> 3)) = o;
            }
          }
          if constexpr (T::s2q) {
            // INT4 stage 2: once every drain warp's BF16 H is in the tile, thread (row, half)
            // requantizes group `half` of its row (Eq. (1) over the group's 128 values,
            // written back in place as 16*q codes in the 4-bit operand order, its scale to
            // s_H); then all are done before the MMAs read the codes and the drains the
            // scales. Both steps meet at a bounded barrier of the 8 drain warps.
            __syncwarp();
            if (lane == 0) mbar_arrive(hq);
            if (!(ok = __all_sync(~0u, wait_on(hq, hq_phase, wc, kPSiteHq)))) break;
            hq_phase ^= 1u;
            if (half < NQ) requant_h_row(hb + half * 32768, row_in, shq + row_in * 2 + half, false, 0, 0);
            __syncwarp();
            if (lane == 0) mbar_arrive(hq);
            if (!(ok = __all_sync(~0u, wait_on(hq, hq_phase, wc, kPSiteHq)))) break;
            hq_phase ^= 1u;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_n(hready_lead, 1);
        }
      }
      if (!ok) break;
      if (T::s2q) {
        // INT4 stage 2: group g2's accumulator (16*q by 16*q codes) scaled by s_V[col] (the
        // scale slot) and s_H[row, g2], into the same sums as the residual
        for (int g2 = 0; g2 < NQ; ++g2) {
          const float shv = shq[row_in * 2 + g2];
          if (g2 == 0)
            if (!(ok = __all_sync(~0u, wait_on(&sfull[q.idx], q.phase, wc, kPSiteDrainScale)))) break;
          if (!(ok = __all_sync(~0u, wait_on(&afull[a.idx], a.phase, wc, kPSiteDrainAcc)))) break;
          tc_fence_after();
          drain128(acc, tmem + lane_addr + a.idx * 256 + half * 128,
                   scl + q.idx * (L::kScaleSlot / 4) + g2 * 256 + half * 128, f2_pack(shv, shv));
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_cluster_n(aempty_lead + a.idx * 8, 1);
            if (g2 == NQ - 1) mbar_arrive(&sempty[q.idx]);
          }
          a.next(2);
          if (g2 == NQ - 1) q.next(kSS);
        }
        if (!ok) break;
      }
      if (!T::res) {
#pragma unroll
        for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
      }
      // ------------------------------------------------------------ epilogue
      if (T::s2) {
        if (!(ok = __all_sync(~0u, wait_on(&afull[a.idx], a.phase, wc, kPSiteDrainAcc)))) break;
        tc_fence_after();
      }
      // Y = bf16(Y_res + Y_lr): Y_res = kDq acc (exact), Y_lr from tensor memory. Each
      // 32-column chunk becomes four 16-byte pieces per row; a transpose within groups of
      // four lanes (four rows) gives each lane one piece of each of the group's rows, so a
      // store writes 64 contiguous bytes of 8 rows instead of 16 bytes of 32 rows.
      const int c0 = half * 128;
      const int64_t row4 = static_cast<int64_t>(it.rb) * 256 + row_half + quarter * 32 + (lane & ~3);
      uint16_t* ycol = args.y + it.ct * 256 + c0 + (lane & 3) * 8;
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        uint32_t v[32];
        if constexpr (T::s2) {
          tmem_ld32(tmem + lane_addr + a.idx * 256 + c0 + c, v);
          tmem_wait_ld();
          if (c == 96) {  // the stage-2 accumulator is read: free it before the last stores
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_n(aempty_lead + a.idx * 8, 1);
            a.next(2);
          }
        }
        uint32_t yw[4][4];  // four pieces of 8 columns, as BF16 pairs
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float yv[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if constexpr (T::s2) yv[k] = acc[c + i + k] * kDq + __uint_as_float(v[i + k]);
            else yv[k] = acc[c + i + k] * kDq;
          }
          yw[i >> 3][0] = bf16x2(yv[0], yv[1]);
          yw[i >> 3][1] = bf16x2(yv[2], yv[3]);
          yw[i >> 3][2] = bf16x2(yv[4], yv[5]);
          yw[i >> 3][3] = bf16x2(yv[6], yv[7]);
        }
        transpose4x4(yw, lane);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (row4 + j < args.b)
            *reinterpret_cast<uint4*>(ycol + (row4 + j) * args.n + c) =
                make_uint4(yw[j][0], yw[j][1], yw[j][2], yw[j][3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // Neither CTA frees its tensor memory or leaves while the peer may still arrive on
  // its barriers or read its shared memory through a pair MMA.
  cluster_sync_startup();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (!f) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<EncodeTiledFn>(p);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

bool encode(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
            uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
            CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Clusters of two CTAs of an instantiation that fit on the current device at once
// (computed once per device and instantiation; 0 if the query fails).
template <int kMode, bool kXB>
int resident_pairs_of() {
  static std::mutex mu;
  static int cache[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    auto kern = twq_pair_kernel<kMode, kXB>;
    int nc = 0;
    int nsm = 0;
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Layout<kXB>::kAlloc) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(nsm & ~1), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = Layout<kXB>::kAlloc;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        nc = 0;
      }
    } else {
      (void)cudaGetLastError();
    }
    cache[dev] = nc > 0 ? nc : 0;
    have[dev] = true;
  }
  return cache[dev];
}

// Contiguous runs of tiles (row-block-major) for `pairs` pairs that minimize the largest
// run's cost in K-group steps: each tile costs its residual groups plus about one step of
// stage 2 and epilogue, and a run pays a stage-1 pass (G steps, cheaper when r <= 128)
// at its start and at every row-block change. An equal split of the tiles can leave
// the slowest pair with two stage-1 passes; when a layer has few tiles per pair (the
// down projection: 3.5) that pass is as large as a tile. Binary search on the cost
// bound with a greedy fill, which is optimal for contiguous runs of positive costs.
void partition_items(int num_items, int col_tiles, int G, bool res, bool h, int r, int pairs,
                     int* bounds) {
  const int64_t tile = 10 * ((res ? G : 0) + 1);
  const int64_t hpass = h ? (r <= 128 ? 6 : 10) * static_cast<int64_t>(G) : 0;
  auto runs_for = [&](int64_t cap, int* out) {
    int runs = 0;
    int64_t cost = 0;
    int start = 0;
    for (int t = 0; t < num_items; ++t) {
      const bool new_rb = t > start && t / col_tiles != (t - 1) / col_tiles;
      int64_t add = tile + (new_rb ? hpass : 0);
      if (t == start) add = tile + hpass;
      if (t > start && cost + add > cap) {
        if (out) out[runs] = start;
        ++runs;
        start = t;
        cost = tile + hpass;
      } else {
        cost += add;
      }
    }
    if (out) out[runs] = start;
    return runs + 1;
  };
  int64_t lo = tile + hpass, hi = (tile + hpass) * static_cast<int64_t>(num_items);
  while (lo < hi) {
    const int64_t mid = lo + (hi - lo) / 2;
    if (runs_for(mid, nullptr) <= pairs) hi = mid; else lo = mid + 1;
  }
  const int used = runs_for(lo, bounds);
  for (int p = used; p <= pairs; ++p) bounds[p] = num_items;  // the rest get no tiles
}

template <int kMode, bool kXB>
cudaError_t launch_pair_mode(const GemmCall& c, cudaStream_t st, unsigned long long wait_ns,
                             int stall) {
  using T = Traits<kMode>;
  using L = Layout<kXB>;
  const twq_weights* w = c.w;
  PairArgs a{};
  a.sx = c.sx;
  a.y = static_cast<uint16_t*>(c.out);
  a.b = c.b;
  a.m = static_cast<int>(w->m);
  a.n = static_cast<int>(w->n);
  a.r = static_cast<int>(w->r);
  a.G = a.m / 128;
  a.col_tiles = a.n / 256;
  a.num_items = static_cast<int>((c.b + 255) / 256) * a.col_tiles;
  a.wait_ns = wait_ns;
  a.stall = stall;
  CUtensorMap m_x{}, m_r{}, m_l1{}, m_l2{}, m_sr{}, m_sl1{}, m_sv{};
  const uint64_t kb = static_cast<uint64_t>(a.m / 2);
  const uint64_t G = static_cast<uint64_t>(a.G);
  constexpr CUtensorMapSwizzle kSw = CU_TENSOR_MAP_SWIZZLE_128B;
  // X: int8 codes, 128 per row and group (one group per copy), or packed nibbles,
  // 128 bytes (two groups) per row and copy; rows beyond b read as zeros.
  bool ok = kXB ? encode(&m_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.xq, a.m, c.b, a.m, 128, 128, kSw)
                : encode(&m_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.xq, kb, c.b, kb, 128, 128, kSw);
  if (T::res) {
    ok = ok && encode(&m_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->rq, kb, a.n, kb, 128, 128, kSw);
    // scales: G x n fp32, 256 columns x 4 groups per copy (groups beyond G read as zeros)
    ok = ok && encode(&m_sr, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->sr, a.n, G,
                      static_cast<uint64_t>(a.n) * 4, 256, 4, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (T::h) {
    ok = ok && encode(&m_l1, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->l1q, kb, a.r, kb, 128, a.r / 2, kSw);
    ok = ok && encode(&m_sl1, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->sl1, a.r, G,
                      static_cast<uint64_t>(a.r) * 4, a.r, 4, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (T::s2) {
    ok = ok && encode(&m_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->l2t, a.r, a.n,
                      static_cast<uint64_t>(a.r) * 2, 64, 128, kSw);
  }
  if (T::s2q) {
    // V: n columns of r/2 bytes (both groups of 128 codes in one 128-byte box; the half
    // beyond r/2 reads as zeros when r = 128), in m_l2's place; s_V: (r/128) x n fp32,
    // 256 columns x 4 groups per copy
    ok = ok && c.l2q && c.sl2q &&
         encode(&m_l2, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.l2q, static_cast<uint64_t>(a.r / 2), a.n,
                static_cast<uint64_t>(a.r / 2), 128, 128, kSw);
    ok = ok && encode(&m_sv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, c.sl2q, a.n,
                      static_cast<uint64_t>(a.r / 128), static_cast<uint64_t>(a.n) * 4, 256, 4,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (!ok) return cudaErrorInvalidValue;
  auto kern = twq_pair_kernel<kMode, kXB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  const int rp = resident_pairs_of<kMode, kXB>();
  if (rp <= 0) return cudaErrorInvalidConfiguration;
  const int pairs = std::min(std::min(rp, a.num_items), kMaxPairs);
  partition_items(a.num_items, a.col_tiles, a.G, T::res, T::h, a.r, pairs, a.bounds);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, m_x, m_r, m_l1, m_l2, m_sr, m_sl1, m_sv, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool kXB>
cudaError_t launch_pair_x(const GemmCall& c, cudaStream_t st) {
  constexpr unsigned long long kWaitNs = 2000000000ull;  // a wait that lasts 2 s is a failure
  switch (c.mode) {
    case kModeFused: return launch_pair_mode<kModeFused, kXB>(c, st, kWaitNs, 0);
    case kModeW4A4: return launch_pair_mode<kModeW4A4, kXB>(c, st, kWaitNs, 0);
    case kModeLowRank: return launch_pair_mode<kModeLowRank, kXB>(c, st, kWaitNs, 0);
    case kModeFusedS2Q:
      if constexpr (!kXB) return launch_pair_mode<kModeFusedS2Q, false>(c, st, kWaitNs, 0);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool pair_eligible(const GemmCall& c) {
  if (c.x != nullptr) return false;
  if (c.mode != kModeFused && c.mode != kModeW4A4 && c.mode != kModeLowRank &&
      c.mode != kModeFusedS2Q)
    return false;
  if (c.a8 && (c.mode == kModeLowRank || c.mode == kModeFusedS2Q)) return false;
  const twq_weights* w = c.w;
  if (w->n % 256 != 0 || w->m < 256 || w->r > kMaxR) return false;
  if (c.mode != kModeW4A4 && w->r <= 0) return false;
  if (c.mode == kModeFusedS2Q && (w->r % 128 != 0 || !c.l2q || !c.sl2q)) return false;
  return c.b > 16;
}

cudaError_t launch_pair(const GemmCall& c, cudaStream_t st) {
  return c.a8 ? launch_pair_x<true>(c, st) : launch_pair_x<false>(c, st);
}

cudaError_t launch_pair_stall_selftest(const GemmCall& c, cudaStream_t st,
                                       unsigned long long wait_ns) {
  return launch_pair_mode<kModeW4A4, false>(c, st, wait_ns, 1);
}

cudaError_t read_and_clear_pair_status(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_pair_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_pair_status, &zero, sizeof(int));
  *code = v;
  return e;
}

}  // namespace twq
