// Tensor-core kernel of the dual-component W4A4 + low-rank linear layer for
// sm_100a (TwinQuant, "Learnable Subspace Decomposition for 4-Bit LLM
// Quantization", §4.3 "Dual-Component Kernel Design" and Fig. 4).
//
// One persistent CTA per SM walks a contiguous run of 128 x BN output tiles
// (row-block major). For each tile:
//   * stage 1 (only when the row block changes): H = Q(X) Q(L1) over all
//     m/128 groups, int32 per group in tensor memory, scaled by
//     sx[i,g] * sl1[g,c] in fp32 and summed in registers; then H -> BF16 into a
//     shared-memory operand tile that later tiles of the same row block reuse
//     (H never goes to HBM);
//   * residual: Y_res = sum_g sx[i,g] sr[g,j] (Q(X)_g Q(R)_g), same scheme;
//   * stage 2: Y_lr = bf16(H) L2 with kind::f16 MMAs (fp32 accumulation);
//   * one epilogue: Y = bf16(Y_res + Y_lr), a single store.
//
// Warp roles (512 threads):
//   warp 0        TMA producer: packed 4-bit code tiles of X and R / L1, BF16
//                 tiles of L2^T, and the per-group weight scales;
//   warp 1        tcgen05.mma issuer (one thread) and TMEM owner;
//   warps 2-7     unpack: 4-bit codes -> int8 in the UMMA 128-byte-swizzle
//                 K-major layout (each byte holds 16*q; the MMA result is 256x
//                 the integer dot product and is rescaled exactly by 2^-8);
//   warps 8-15    drain: per-group tensor-memory loads, fp32 scaling and
//                 accumulation, H -> BF16, epilogue.
// Inside every 16-byte chunk the unpack writes the even-index codes first and
// the odd-index codes second; A and B use the same order, so every product
// still pairs the same k and the per-group integer sums are unchanged.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "sm100_ptx.cuh"
#include "twq_eq1.cuh"
#include "twq_internal.h"
#include "twq_hrequant.cuh"

namespace twq {

__device__ int g_device_status;

namespace {

constexpr int kThreads = 512;

constexpr int kBM = 128;
constexpr int kPackedStages = 4;
constexpr int kUnpackedStages = 2;
constexpr int kScaleSlots = 8;
constexpr int kAccBufs = 4;     // TMEM accumulator buffers (BN columns each)
constexpr int kHChunk = 128;  // H columns per stage-1 pass
constexpr int kMaxRank = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a wait that lasts 2 s is a failure

template <int kMode>
struct ModeTraits {
  static constexpr bool res = kMode == kModeFused || kMode == kModeW4A4 || kMode == kModeResF32 ||
                              kMode == kModeFusedS2Q;
  static constexpr bool h = kMode == kModeFused || kMode == kModeLowRank || kMode == kModeHOnly ||
                            kMode == kModeFusedS2Q;
  // The INT4 stage 2: H requantized on chip, multiplied by 4-bit L2 codes as r/128 more
  // K groups of the residual accumulation (kind::i8), not by the BF16 stage 2.
  static constexpr bool s2q = kMode == kModeFusedS2Q;
  static constexpr bool s2 = kMode == kModeFused || kMode == kModeLowRank || kMode == kModeS2F32;
  static constexpr bool h_global = kMode == kModeS2F32;
  static constexpr bool out_f32 = kMode == kModeResF32 || kMode == kModeS2F32;
  static constexpr bool out_h = kMode == kModeHOnly;
};

// kA8 (W4A8): the X tile is 128 rows x 128 int8 codes, TMA-loaded with the 128-byte
// swizzle straight into the packed slot, where the MMA reads it (no unpack); three
// stages of 24 KB instead of four of 16 KB keep the budget.
template <int BN, bool kA8 = false>
struct SmemLayout {
  static constexpr int kStages = kA8 ? 3 : kPackedStages;
  static constexpr int kSlotA = kA8 ? 16384 : 8192;  // 128 rows x 128 int8, or x 64 packed bytes
  static constexpr int kSlot = (kSlotA + BN * 64) > BN * 128 ? (kSlotA + BN * 64) : BN * 128;
  static constexpr int kUA = 16384;   // 128 rows x 128 int8
  static constexpr int kUB = BN * 128;
  static constexpr int kUStage = kUA + kUB;
  static constexpr int kHb = kBM * kMaxRank * 2;  // up to 4 K-chunks of 128 x 64 BF16
  static constexpr int kScaleSlot = BN * 4;
  static constexpr int kOffSlots = 0;
  static constexpr int kOffU = kOffSlots + kStages * kSlot;
  static constexpr int kOffHb = kOffU + kUnpackedStages * kUStage;
  static constexpr int kOffScale = kOffHb + kHb;
  static constexpr int kOffShq = kOffScale + kScaleSlots * kScaleSlot;  // s_H: 128 rows x 2 groups
  static constexpr int kOffBar = kOffShq + kBM * 2 * 4;
  static constexpr int kNumBars =
      2 * kStages + 2 * kUnpackedStages + 2 * kAccBufs + 2 * kScaleSlots + 5;
  static constexpr int kBytes = kOffBar + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024 bytes
  static constexpr int kTmemCols = kAccBufs * BN;  // accumulator buffers
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
  static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM allocation must be a power of 2");
  static_assert(!kA8 || kSlot % 1024 == 0, "a 128-byte-swizzle TMA tile starts on 1 KB");
};

struct GemmArgs {
  const float* sx;
  const float* sr;
  const float* sl1;
  void* out;
  int64_t b;
  int m, n, r, G;
  int row_blocks, col_tiles, num_tiles;
  int tiles_per_rb;  // tiles (or, for CTA pairs, pairs of column tiles) per row block
  int r_pad;  // stage-2 K extent: r rounded up to 64
  int h_box;  // rows of the L1 TMA box: min(r, 128)
  const float* sl2q;  // INT4 stage 2: scales of the 4-bit L2 codes, (r/128) x n
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

__device__ __forceinline__ void record_failure(int site) {
  atomicCAS(&g_device_status, 0, site);
}

// Bounded wait on a barrier phase. Returns false if the CTA is aborting or the
// wait ran out (then it records `site` and raises the abort flag).
__device__ __noinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      record_failure(site);
      *abort_flag = 1;
      return false;
    }
  }
}

// wait_bar with the first probe inline, for the single-thread producer and MMA
// roles, where the phase has often completed already and a call costs more than
// the probe.
__device__ __forceinline__ bool wait_fast(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int site) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bar(bar, parity, abort_flag, site);
}

// Bounded wait with cluster-scope acquire, for barriers that complete on a peer
// CTA's arrivals or stores.
__device__ __noinline__ bool wait_bar_cluster(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int site) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      record_failure(site);
      *abort_flag = 1;
      return false;
    }
  }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Offset of 16-byte chunk `c` of row `row` in a K-major 128-byte-swizzle tile.
__device__ __forceinline__ uint32_t sw128_offset(int row, int c) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((c ^ (row & 7)) << 4));
}

// 4-bit codes (rows x 64 bytes, dense) -> int8 (rows x 128 bytes, swizzled), 16*q per byte.
// A thread of the 192 unpack threads takes the 16-byte items tid, tid + 192 and
// tid + 384 of a 128-row tile (an item: 16 packed bytes of one row, two output
// chunks). The offsets depend only on the thread, so they are computed once.
constexpr int kUnpackThreads = 192;
struct UnpackPlan {
  uint32_t src[3];     // byte offset of the item in the packed tile
  uint32_t dst0[3];    // swizzled offsets of its two output chunks
  uint32_t dst1[3];
  int row[3];          // tile row of the item (>= 128: no item)
};

__device__ __forceinline__ UnpackPlan unpack_plan(int tid) {
  UnpackPlan p;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int e = tid + i * kUnpackThreads;
    const int row = e >> 2;
    const int c = (e & 3) * 2;
    p.row[i] = row;
    p.src[i] = static_cast<uint32_t>(e * 16);
    p.dst0[i] = sw128_offset(row & 127, c);
    p.dst1[i] = sw128_offset(row & 127, c + 1);
  }
  return p;
}

// Unpacks the first `rows` rows (<= 128) of a tile with the thread's plan; all
// loads are issued before any store so the shared-memory latencies overlap.
// kNatural: element order within each 16-byte chunk (to pair with int8 X codes
// loaded as they are, W4A8), two byte permutes per 8 output bytes; else even
// elements first, the order both 4-bit operands share.
template <bool kNatural = false>
__device__ __forceinline__ void unpack_tile(const uint8_t* src, uint8_t* dst, int rows,
                                            const UnpackPlan& p) {
  uint4 w[3];
#pragma unroll
  for (int i = 0; i < 3; ++i)
    if (p.row[i] < rows) w[i] = *reinterpret_cast<const uint4*>(src + p.src[i]);
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    if (p.row[i] < rows) {
      uint4 o0, o1;
      o0.x = (w[i].x << 4) & 0xF0F0F0F0u;  // 16 x elements 0, 2, 4, 6 of the word
      o0.y = w[i].x & 0xF0F0F0F0u;         // 16 x elements 1, 3, 5, 7
      o0.z = (w[i].y << 4) & 0xF0F0F0F0u;
      o0.w = w[i].y & 0xF0F0F0F0u;
      o1.x = (w[i].z << 4) & 0xF0F0F0F0u;
      o1.y = w[i].z & 0xF0F0F0F0u;
      o1.z = (w[i].w << 4) & 0xF0F0F0F0u;
      o1.w = w[i].w & 0xF0F0F0F0u;
      if constexpr (kNatural) {
        const uint4 e0 = o0, e1 = o1;
        o0 = make_uint4(__byte_perm(e0.x, e0.y, 0x5140), __byte_perm(e0.x, e0.y, 0x7362),
                        __byte_perm(e0.z, e0.w, 0x5140), __byte_perm(e0.z, e0.w, 0x7362));
        o1 = make_uint4(__byte_perm(e1.x, e1.y, 0x5140), __byte_perm(e1.x, e1.y, 0x7362),
                        __byte_perm(e1.z, e1.w, 0x5140), __byte_perm(e1.z, e1.w, 0x7362));
      }
      *reinterpret_cast<uint4*>(dst + p.dst0[i]) = o0;
      *reinterpret_cast<uint4*>(dst + p.dst1[i]) = o1;
    }
  }
}

__device__ __forceinline__ void copy_smem(const uint8_t* src, uint8_t* dst, int bytes, int tid,
                                          int nthreads) {
  for (int off = tid * 16; off < bytes; off += nthreads * 16)
    *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(src + off);
}

// acc[j] += float(I[j]) * sc[j] * sx for this thread's lane and ncols columns
// (ncols % 8 == 0, <= 64) of the int32 accumulator at taddr.
__device__ __forceinline__ void drain_group(float (&acc)[64], uint32_t taddr, int ncols,
                                            const float* sc, float sx) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    if (h * 16 < ncols) {
      uint32_t v[16];
      uint32_t t0[8], t1[8];
      tmem_ld8(taddr + h * 16, t0);
      if (h * 16 + 8 < ncols) tmem_ld8(taddr + h * 16 + 8, t1);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        v[k] = t0[k];
        v[k + 8] = t1[k];
      }
#pragma unroll
      for (int c = 0; c < 16; c += 4)
        if (h * 16 + c < ncols) {
          const float4 s4 = *reinterpret_cast<const float4*>(sc + h * 16 + c);
          const int j = h * 16 + c;
          acc[j + 0] = fmaf(static_cast<float>(static_cast<int32_t>(v[c + 0])) * s4.x, sx, acc[j + 0]);
          acc[j + 1] = fmaf(static_cast<float>(static_cast<int32_t>(v[c + 1])) * s4.y, sx, acc[j + 1]);
          acc[j + 2] = fmaf(static_cast<float>(static_cast<int32_t>(v[c + 2])) * s4.z, sx, acc[j + 2]);
          acc[j + 3] = fmaf(static_cast<float>(static_cast<int32_t>(v[c + 3])) * s4.w, sx, acc[j + 3]);
        }
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct TileInfo {
  int rb, ct;
  bool need_h;
};

// Work item t of a CTA's run: a tile, or for a CTA pair a pair of adjacent
// column tiles of one row block, of which CTA `prank` takes one.
__device__ __forceinline__ TileInfo tile_info(const GemmArgs& a, int t, int t_begin, bool has_h,
                                              int pair_stride, int prank) {
  TileInfo ti;
  ti.rb = t / a.tiles_per_rb;
  ti.ct = (t % a.tiles_per_rb) * pair_stride + prank;
  ti.need_h = has_h && (t == t_begin || (t - 1) / a.tiles_per_rb != ti.rb);
  return ti;
}

// kPair: a cluster of two CTAs works on the two column tiles of one pair at a
// time; CTA k computes H columns [k r/2, (k+1) r/2) of the row block and stores
// its BF16 slice into both CTAs' H operand tiles, so H is computed once per pair.
// kA8: W4A8, X as int8 codes (q_max = 127) read by the MMA where TMA put them.
template <int kMode, int BN, bool kPair, bool kA8>
__global__ void __launch_bounds__(kThreads, 1)
    twq_gemm_kernel(const __grid_constant__ CUtensorMap tm_xq,
                    const __grid_constant__ CUtensorMap tm_rq,
                    const __grid_constant__ CUtensorMap tm_l1q,
                    const __grid_constant__ CUtensorMap tm_l2t,
                    const __grid_constant__ CUtensorMap tm_h, const GemmArgs args) {
  using L = SmemLayout<BN, kA8>;
  using T = ModeTraits<kMode>;
  // The weight operand holds 16*q (4-bit codes); X holds 16*q (W4A4) or q (W4A8):
  // an accumulator is 2^8 (2^4) times the group's integer dot product.
  constexpr float kDq = kA8 ? 0.0625f : 0.00390625f;
  constexpr int kStages = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_abort;
  uint8_t* smem = align1024(smem_raw);
  uint8_t* slots = smem + L::kOffSlots;
  uint8_t* ustg = smem + L::kOffU;
  uint8_t* hb = smem + L::kOffHb;
  float* scl = reinterpret_cast<float*>(smem + L::kOffScale);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* ufull = empty + kStages;
  uint64_t* uempty = ufull + kUnpackedStages;
  uint64_t* acc_full = uempty + kUnpackedStages;
  uint64_t* acc_empty = acc_full + kAccBufs;
  uint64_t* sc_full = acc_empty + kAccBufs;
  uint64_t* sc_empty = sc_full + kScaleSlots;
  uint64_t* hb_ready = sc_empty + kScaleSlots;
  uint64_t* hb_free = hb_ready + 1;
  uint64_t* mma_done = hb_free + 1;
  uint64_t* peer_free = mma_done + 1;  // kPair: the peer may overwrite its slice of our H
  uint64_t* hq = mma_done + 2;         // INT4 stage 2: every drain warp's BF16 H is in hb
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 3);
  float* shq = reinterpret_cast<float*>(smem + L::kOffShq);  // s_H[row * 2 + group of r]
  volatile int* abort_flag = &s_abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = args.G;
  // H chunks this CTA computes per row block: r in chunks of 128, or for a pair
  // one chunk of r/2 columns at row offset prank * r/2 of L1
  const int prank = kPair ? static_cast<int>(cluster_rank()) : 0;
  const int HC = !T::h ? 0 : (kPair ? 1 : (args.r + kHChunk - 1) / kHChunk);
  auto h_row0 = [&](int hc) { return kPair ? prank * (args.r / 2) : hc * kHChunk; };
  auto h_cols = [&](int hc) { return kPair ? args.r / 2 : min(kHChunk, args.r - hc * kHChunk); };
  const int KC = args.r_pad / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kA8 ? 7 : 6);  // the unpack warps (+ the MMA, which reads X there)
    }
    for (int i = 0; i < kUnpackedStages; ++i) {
      mbar_init(&ufull[i], 6);
      mbar_init(&uempty[i], 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 8);
    }
    for (int i = 0; i < kScaleSlots; ++i) {
      mbar_init(&sc_full[i], 1);
      mbar_init(&sc_empty[i], 8);
    }
    mbar_init(hb_ready, T::h_global ? 1 : 8);
    mbar_init(hb_free, 1);
    mbar_init(mma_done, 1);
    mbar_init(peer_free, 8);  // each of the peer's 8 drain warps
    mbar_init(hq, 8);
    s_abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tm_xq);
    if (T::res) tma_prefetch_desc(&tm_rq);
    if (T::h) tma_prefetch_desc(&tm_l1q);
    if (T::s2) tma_prefetch_desc(&tm_l2t);
    if (T::h_global) tma_prefetch_desc(&tm_h);
  }
  // Zero the K padding [r, r_pad) of the on-chip H operand (stage 2 reads it).
  if (T::s2 && !T::h_global) {
    const int pad_units = (args.r_pad - args.r) / 8;
    for (int e = threadIdx.x; e < kBM * pad_units; e += kThreads) {
      const int row = e / pad_units;
      const int col = args.r + (e % pad_units) * 8;
      *reinterpret_cast<uint4*>(hb + (col >> 6) * 16384 + sw128_offset(row, (col & 63) >> 3)) =
          make_uint4(0, 0, 0, 0);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, L::kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // Runs of work items: per CTA, or per CTA pair (both CTAs of a pair take the same run).
  const int unit = kPair ? static_cast<int>(blockIdx.x) / 2 : static_cast<int>(blockIdx.x);
  const int units = kPair ? static_cast<int>(gridDim.x) / 2 : static_cast<int>(gridDim.x);
  const int t_begin = static_cast<int>((int64_t)unit * args.num_tiles / units);
  const int t_end = static_cast<int>((int64_t)(unit + 1) * args.num_tiles / units);
  constexpr int kPairStride = kPair ? 2 : 1;
  // The peer's barriers are initialized before any remote store or arrive.
  if (kPair) cluster_sync_startup();

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      Ring s, q;
      uint32_t hb_phase = 0;
      bool hb_pend = false;
      bool pend[kStages] = {};
      uint32_t pend_phase[kStages];
      bool spend[kScaleSlots] = {};
      uint32_t spend_phase[kScaleSlots];
      bool ok = true;
      for (int t = t_begin; t < t_end && ok; ++t) {
        const TileInfo ti = tile_info(args, t, t_begin, T::h, kPairStride, prank);
        const int row0 = ti.rb * kBM;
        const int n0 = ti.ct * BN;
        if (ti.need_h) {
          for (int hc = 0; hc < HC && ok; ++hc) {
            const int nh = h_cols(hc);
            for (int g = 0; g < G; ++g) {
              if (!(ok = wait_fast(&empty[s.idx], s.phase ^ 1u, abort_flag, kSiteProducerEmpty)))
                break;
              uint8_t* slot = slots + s.idx * L::kSlot;
              mbar_arrive_expect_tx(&full[s.idx], L::kSlotA + args.h_box * 64);
              tma_load_2d(slot, &tm_xq, &full[s.idx], g * (kA8 ? 128 : 64), row0);
              tma_load_2d(slot + L::kSlotA, &tm_l1q, &full[s.idx], g * 64, h_row0(hc));
              pend[s.idx] = true;
              pend_phase[s.idx] = s.phase;
              s.next(kStages);
              if (!(ok = wait_fast(&sc_empty[q.idx], q.phase ^ 1u, abort_flag,
                                  kSiteProducerScaleEmpty)))
                break;
              mbar_arrive_expect_tx(&sc_full[q.idx], nh * 4);
              bulk_load(scl + q.idx * BN, args.sl1 + (int64_t)g * args.r + h_row0(hc), nh * 4,
                        &sc_full[q.idx]);
              spend[q.idx] = true;
              spend_phase[q.idx] = q.phase;
              q.next(kScaleSlots);
            }
          }
        }
        if (T::res && ok) {
          for (int g = 0; g < G; ++g) {
            if (!(ok = wait_fast(&empty[s.idx], s.phase ^ 1u, abort_flag, kSiteProducerEmpty)))
              break;
            uint8_t* slot = slots + s.idx * L::kSlot;
            mbar_arrive_expect_tx(&full[s.idx], L::kSlotA + BN * 64);
            tma_load_2d(slot, &tm_xq, &full[s.idx], g * (kA8 ? 128 : 64), row0);
            tma_load_2d(slot + L::kSlotA, &tm_rq, &full[s.idx], g * 64, n0);
            pend[s.idx] = true;
            pend_phase[s.idx] = s.phase;
            s.next(kStages);
            if (!(ok = wait_fast(&sc_empty[q.idx], q.phase ^ 1u, abort_flag,
                                kSiteProducerScaleEmpty)))
              break;
            mbar_arrive_expect_tx(&sc_full[q.idx], BN * 4);
            bulk_load(scl + q.idx * BN, args.sr + (int64_t)g * args.n + n0, BN * 4,
                      &sc_full[q.idx]);
            spend[q.idx] = true;
            spend_phase[q.idx] = q.phase;
            q.next(kScaleSlots);
          }
        }
        if (T::s2q && ok) {
          // INT4 stage 2: the tile's 4-bit L2 codes, one group of 128 along r per step
          // (the A operand, the requantized H, is already on chip), and their scales
          for (int g2 = 0; g2 < args.r / 128; ++g2) {
            if (!(ok = wait_fast(&empty[s.idx], s.phase ^ 1u, abort_flag, kSiteProducerEmpty)))
              break;
            uint8_t* slot = slots + s.idx * L::kSlot;
            mbar_arrive_expect_tx(&full[s.idx], BN * 64);
            tma_load_2d(slot + L::kSlotA, &tm_l2t, &full[s.idx], g2 * 64, n0);
            pend[s.idx] = true;
            pend_phase[s.idx] = s.phase;
            s.next(kStages);
            if (!(ok = wait_fast(&sc_empty[q.idx], q.phase ^ 1u, abort_flag,
                                kSiteProducerScaleEmpty)))
              break;
            mbar_arrive_expect_tx(&sc_full[q.idx], BN * 4);
            bulk_load(scl + q.idx * BN, args.sl2q + (int64_t)g2 * args.n + n0, BN * 4,
                      &sc_full[q.idx]);
            spend[q.idx] = true;
            spend_phase[q.idx] = q.phase;
            q.next(kScaleSlots);
          }
        }
        if (T::s2 && ok) {
          if (T::h_global) {
            if (!(ok = wait_fast(hb_free, hb_phase ^ 1u, abort_flag, kSiteProducerHbFree))) break;
            mbar_arrive_expect_tx(hb_ready, KC * 16384);
            for (int kc = 0; kc < KC; ++kc)
              tma_load_2d(hb + kc * 16384, &tm_h, hb_ready, kc * 64, row0);
            hb_pend = true;
            hb_phase ^= 1u;
          }
          for (int kc = 0; kc < KC; ++kc) {
            if (!(ok = wait_fast(&empty[s.idx], s.phase ^ 1u, abort_flag, kSiteProducerEmpty)))
              break;
            mbar_arrive_expect_tx(&full[s.idx], BN * 128);
            tma_load_2d(slots + s.idx * L::kSlot, &tm_l2t, &full[s.idx], kc * 64, n0);
            pend[s.idx] = true;
            pend_phase[s.idx] = s.phase;
            s.next(kStages);
          }
        }
      }
      if (!ok) {
        // Aborting: let the copies already issued land before the CTA exits.
        int dummy = 0;
        volatile int* never = &dummy;
        for (int i = 0; i < kStages; ++i)
          if (pend[i]) wait_fast(&full[i], pend_phase[i], never, kSiteFinal);
        for (int i = 0; i < kScaleSlots; ++i)
          if (spend[i]) wait_fast(&sc_full[i], spend_phase[i], never, kSiteFinal);
        if (T::h_global && hb_pend) wait_fast(hb_ready, hb_phase ^ 1u, never, kSiteFinal);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      Ring u, a, s;  // s: the packed slot of each step (W4A8: X is read there)
      uint32_t hb_phase = 0;
      bool ok = true;
      const uint32_t ua0 = smem_u32(ustg);
      const uint32_t hb0 = smem_u32(hb);
      const uint32_t slot0 = smem_u32(slots);
      // W4A8: the step's packed slot is released by the unpack warps and by this commit
      auto release_slot = [&]() {
        if constexpr (kA8) mma_commit(&empty[s.idx]);
        s.next(kStages);
      };
      for (int t = t_begin; t < t_end && ok; ++t) {
        const TileInfo ti = tile_info(args, t, t_begin, T::h, kPairStride, prank);
        if (ti.need_h) {
          for (int hc = 0; hc < HC && ok; ++hc) {
            const int nh = h_cols(hc);
            const uint32_t idesc = idesc_i8(nh);
            for (int g = 0; g < G; ++g) {
              if (!(ok = wait_fast(&ufull[u.idx], u.phase, abort_flag, kSiteMmaFull))) break;
              if (!(ok = wait_fast(&acc_empty[a.idx], a.phase ^ 1u, abort_flag, kSiteMmaAccEmpty)))
                break;
              tc_fence_after();
              const uint32_t d = tmem_base + a.idx * BN;
              const uint64_t da = kA8 ? smem_desc_sw128(slot0 + s.idx * L::kSlot)
                                      : smem_desc_sw128(ua0 + u.idx * L::kUStage);
              const uint64_t db = smem_desc_sw128(ua0 + u.idx * L::kUStage + L::kUA);
#pragma unroll
              for (int k = 0; k < 4; ++k) mma_i8(d, da + 2 * k, db + 2 * k, idesc, k > 0);
              mma_commit(&uempty[u.idx]);
              mma_commit(&acc_full[a.idx]);
              release_slot();
              u.next(kUnpackedStages);
              a.next(kAccBufs);
            }
          }
        }
        if (T::res && ok) {
          const uint32_t idesc = idesc_i8(BN);
          for (int g = 0; g < G; ++g) {
            if (!(ok = wait_fast(&ufull[u.idx], u.phase, abort_flag, kSiteMmaFull))) break;
            if (!(ok = wait_fast(&acc_empty[a.idx], a.phase ^ 1u, abort_flag, kSiteMmaAccEmpty)))
              break;
            tc_fence_after();
            const uint32_t d = tmem_base + a.idx * BN;
            const uint64_t da = kA8 ? smem_desc_sw128(slot0 + s.idx * L::kSlot)
                                    : smem_desc_sw128(ua0 + u.idx * L::kUStage);
            const uint64_t db = smem_desc_sw128(ua0 + u.idx * L::kUStage + L::kUA);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_i8(d, da + 2 * k, db + 2 * k, idesc, k > 0);
            mma_commit(&uempty[u.idx]);
            mma_commit(&acc_full[a.idx]);
            release_slot();
            u.next(kUnpackedStages);
            a.next(kAccBufs);
          }
        }
        if (T::s2q && ok) {
          // INT4 stage 2: A = the requantized H of group g2 (int8 16*q, written by the
          // drain warps over the first 16 KB of H's BF16 columns [128 g2, 128 g2 + 128)),
          // B = the unpacked 4-bit L2 codes
          if (ti.need_h) {
            if (kPair) {  // half of the codes came from the peer's st.async stores
              if (!(ok = wait_bar_cluster(hb_ready, hb_phase, abort_flag, kSiteMmaHb))) break;
              fence_proxy_async_smem();
            } else if (!(ok = wait_fast(hb_ready, hb_phase, abort_flag, kSiteMmaHb))) {
              break;
            }
            hb_phase ^= 1u;
          }
          const uint32_t idesc = idesc_i8(BN);
          for (int g2 = 0; g2 < args.r / 128; ++g2) {
            if (!(ok = wait_fast(&ufull[u.idx], u.phase, abort_flag, kSiteMmaFull))) break;
            if (!(ok = wait_fast(&acc_empty[a.idx], a.phase ^ 1u, abort_flag, kSiteMmaAccEmpty)))
              break;
            tc_fence_after();
            const uint32_t d = tmem_base + a.idx * BN;
            const uint64_t da = smem_desc_sw128(hb0 + g2 * 32768);
            const uint64_t db = smem_desc_sw128(ua0 + u.idx * L::kUStage + L::kUA);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_i8(d, da + 2 * k, db + 2 * k, idesc, k > 0);
            mma_commit(&uempty[u.idx]);
            mma_commit(&acc_full[a.idx]);
            release_slot();
            u.next(kUnpackedStages);
            a.next(kAccBufs);
          }
        }
        if (T::s2 && ok) {
          if (ti.need_h || T::h_global) {
            if (kPair) {
              // half of H came from the peer's st.async stores
              if (!(ok = wait_bar_cluster(hb_ready, hb_phase, abort_flag, kSiteMmaHb))) break;
              fence_proxy_async_smem();
            } else if (!(ok = wait_fast(hb_ready, hb_phase, abort_flag, kSiteMmaHb))) {
              break;
            }
            hb_phase ^= 1u;
          }
          if (!(ok = wait_fast(&acc_empty[a.idx], a.phase ^ 1u, abort_flag, kSiteMmaAccEmpty)))
            break;
          const uint32_t idesc = idesc_bf16(BN);
          const uint32_t d = tmem_base + a.idx * BN;
          for (int kc = 0; kc < KC; ++kc) {
            if (!(ok = wait_fast(&ufull[u.idx], u.phase, abort_flag, kSiteMmaFull))) break;
            tc_fence_after();
            const uint64_t da = smem_desc_sw128(hb0 + kc * 16384);
            const uint64_t db = smem_desc_sw128(ua0 + u.idx * L::kUStage + L::kUA);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16(d, da + 2 * k, db + 2 * k, idesc, (kc | k) != 0);
            mma_commit(&uempty[u.idx]);
            release_slot();
            u.next(kUnpackedStages);
          }
          if (!ok) break;
          mma_commit(&acc_full[a.idx]);
          if (T::h_global) mma_commit(hb_free);
          a.next(kAccBufs);
        }
      }
      // All MMAs issued by this thread are complete before TMEM is released.
      mma_commit(mma_done);
      int dummy = 0;
      wait_fast(mma_done, 0, &dummy, kSiteFinal);
    }
  } else if (warp >= 2 && warp < 8) {
    // --------------------------------------------------------------- unpack
    static_assert(kBM == 128 && BN == 128, "the unpack plan covers 128-row tiles");
    const int tid = threadIdx.x - 64;
    const UnpackPlan plan = unpack_plan(tid);
    Ring s, u;
    bool ok = true;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const TileInfo ti = tile_info(args, t, t_begin, T::h, kPairStride, prank);
      const int n_h = ti.need_h ? HC * G : 0;
      const int n_res = T::res ? G : 0;
      const int n_q = T::s2q ? args.r / 128 : 0;
      const int n_l2 = T::s2 ? KC : 0;
      for (int step = 0; step < n_h + n_res + n_q + n_l2; ++step) {
        if (!(ok = wait_bar(&full[s.idx], s.phase, abort_flag, kSiteUnpackFull))) break;
        if (!(ok = wait_bar(&uempty[u.idx], u.phase ^ 1u, abort_flag, kSiteUnpackEmpty))) break;
        const uint8_t* src = slots + s.idx * L::kSlot;
        uint8_t* dst = ustg + u.idx * L::kUStage;
        if (step < n_h + n_res) {
          int brows = BN;
          if (step < n_h) {
            const int hc = step / G;
            brows = h_cols(hc);
          }
          if constexpr (!kA8) unpack_tile(src, dst, kBM, plan);  // W4A8: the MMA reads X in place
          unpack_tile<kA8>(src + L::kSlotA, dst + L::kUA, brows, plan);
        } else if (step < n_h + n_res + n_q) {  // INT4 stage 2: only the L2 codes (B)
          unpack_tile(src + L::kSlotA, dst + L::kUA, BN, plan);
        } else {
          copy_smem(src, dst + L::kUA, BN * 128, tid, 192);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ufull[u.idx]);
          mbar_arrive(&empty[s.idx]);
        }
        s.next(kStages);
        u.next(kUnpackedStages);
      }
    }
  } else if (warp >= 8) {
    // ---------------------------------------------------------------- drain
    const int dw = warp - 8;
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    const int half = dw >> 2;      // which half of the tile's columns
    const int row_in = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    Ring a, q;
    uint32_t peer_phase = 0;  // kPair: phase of peer_free for the next H slice
    uint32_t hq_phase = 0;    // INT4 stage 2: phases of hq and (as a consumer) of hb_ready
    uint32_t hbq_phase = 0;
    bool ok = true;
    float acc[64];
    for (int t = t_begin; t < t_end && ok; ++t) {
      const TileInfo ti = tile_info(args, t, t_begin, T::h, kPairStride, prank);
      const int64_t row = static_cast<int64_t>(ti.rb) * kBM + row_in;
      const bool row_ok = row < args.b;
      const float* sx_row = args.sx + (row_ok ? row : 0) * G;
      const int n0 = ti.ct * BN;
      if (ti.need_h) {
        for (int hc = 0; hc < HC && ok; ++hc) {
          const int nh = h_cols(hc);
          const int ncols = nh / 2;
          const int c0 = half * ncols;
#pragma unroll
          for (int j = 0; j < 64; ++j) acc[j] = 0.0f;
          float sx0 = row_ok ? __ldg(sx_row) : 0.0f;
          float sx1 = (row_ok && G > 1) ? __ldg(sx_row + 1) : 0.0f;
          for (int g = 0; g < G; ++g) {
            const float sx = sx0;
            sx0 = sx1;
            sx1 = (row_ok && g + 2 < G) ? __ldg(sx_row + g + 2) : 0.0f;
            if (!(ok = wait_bar(&acc_full[a.idx], a.phase, abort_flag, kSiteDrainAccFull))) break;
            // The first stage-1 accumulator of a row block implies that every earlier MMA of
            // this CTA, stage 2 of the previous row block included, has completed, and this
            // warp has finished the previous row block (INT4 stage 2: its reads of the
            // peer's scales). Once all 8 drain warps say so, the peer may overwrite its
            // slice of our H tile and its scales.
            if (kPair && hc == 0 && g == 0 && lane == 0)
              mbar_arrive_peer(map_peer(smem_u32(peer_free), static_cast<uint32_t>(prank ^ 1)));
            tc_fence_after();
            if (!(ok = wait_bar(&sc_full[q.idx], q.phase, abort_flag, kSiteDrainScaleFull))) break;
            drain_group(acc, tmem_base + lane_addr + a.idx * BN + c0, ncols, scl + q.idx * BN + c0,
                        sx);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&acc_empty[a.idx]);
              mbar_arrive(&sc_empty[q.idx]);
            }
            a.next(kAccBufs);
            q.next(kScaleSlots);
          }
          if (!ok) break;
          // A pair stores its slice into the peer's H tile too, once the peer's stage 2 no
          // longer reads it.
          if (kPair) {
            if (!(ok = wait_bar_cluster(peer_free, peer_phase, abort_flag, kSiteDrainPeerFree)))
              break;
            peer_phase ^= 1u;
          }
          // H chunk complete: 2^-8 undoes the 16x16 code scaling of the unpack.
#pragma unroll
          for (int j = 0; j < 64; j += 8) {
            if (j < ncols) {
              uint4 o;
              o.x = pack_bf16x2(acc[j + 0] * kDq, acc[j + 1] * kDq);
              o.y = pack_bf16x2(acc[j + 2] * kDq, acc[j + 3] * kDq);
              o.z = pack_bf16x2(acc[j + 4] * kDq, acc[j + 5] * kDq);
              o.w = pack_bf16x2(acc[j + 6] * kDq, acc[j + 7] * kDq);
              const int col = h_row0(hc) + c0 + j;
              if (T::out_h) {
                if (row_ok)
                  *reinterpret_cast<uint4*>(static_cast<uint16_t*>(args.out) + row * args.r +
                                            col) = o;
              } else {
                uint8_t* dst = hb + (col >> 6) * 16384 + sw128_offset(row_in, (col & 63) >> 3);
                *reinterpret_cast<uint4*>(dst) = o;
                if (kPair && !T::s2q) {  // INT4 stage 2: the codes are pushed instead
                  const uint32_t peer = static_cast<uint32_t>(prank ^ 1);
                  st_async_peer_v4u(map_peer(smem_u32(dst), peer), o,
                                    map_peer(smem_u32(hb_ready), peer));
                }
              }
            }
          }
        }
        if (!ok) break;
        if constexpr (T::s2q) {
          // INT4 stage 2: Eq. (1) on bf16(H) per row and group of 128 along r. A group's
          // columns come from both halves' warps, so every drain warp's BF16 H must be in
          // hb first (a bounded barrier, so that an aborting warp cannot strand the others).
          __syncwarp();
          if (lane == 0) mbar_arrive(hq);
          if (!(ok = wait_bar(hq, hq_phase, abort_flag, kSiteDrainHq))) break;
          hq_phase ^= 1u;
          // Thread (row, half) takes group `half` of its row: it reads the group's 128 BF16
          // values (16 pieces of 8) into registers, then writes the 16*q codes over the
          // group's first 16 KB (only this thread touches these bytes of this row).
          if (kPair) {
            // a pair (r = 256): this CTA's H columns are group prank of r; it requantizes
            // them and stores the codes and scales into both CTAs
            const uint32_t peer = static_cast<uint32_t>(prank ^ 1);
            if (half == 0)
              requant_h_row(hb + prank * 32768, row_in, shq + row_in * 2 + prank, true, peer,
                            map_peer(smem_u32(hb_ready), peer));
          } else if (half < args.r / 128) {
            requant_h_row(hb + half * 32768, row_in, shq + row_in * 2 + half, false, 0, 0);
          }
        }
        if (!T::out_h) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // For a pair, one arrival also registers the bytes the peer stores into our
            // H tile (its r/2 columns of the 128 rows, BF16).
            if (kPair && dw == 0)  // BF16 slice (r/2 columns) or, INT4 stage 2, codes + scales
              mbar_arrive_expect_tx(hb_ready, T::s2q ? static_cast<uint32_t>(kBM * (128 + 4))
                                                     : static_cast<uint32_t>(kBM * (args.r / 2) * 2));
            else
              mbar_arrive(hb_ready);
          }
        }
      }
      if (T::out_h) continue;
      const int ncols = BN / 2;
      const int c0 = half * ncols;
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.0f;
      if (T::res) {
        float sx0 = row_ok ? __ldg(sx_row) : 0.0f;
        float sx1 = (row_ok && G > 1) ? __ldg(sx_row + 1) : 0.0f;
        for (int g = 0; g < G; ++g) {
          const float sx = sx0;
          sx0 = sx1;
          sx1 = (row_ok && g + 2 < G) ? __ldg(sx_row + g + 2) : 0.0f;
          if (!(ok = wait_bar(&acc_full[a.idx], a.phase, abort_flag, kSiteDrainAccFull))) break;
          tc_fence_after();
          if (!(ok = wait_bar(&sc_full[q.idx], q.phase, abort_flag, kSiteDrainScaleFull))) break;
          drain_group(acc, tmem_base + lane_addr + a.idx * BN + c0, ncols, scl + q.idx * BN + c0,
                      sx);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&acc_empty[a.idx]);
            mbar_arrive(&sc_empty[q.idx]);
          }
          a.next(kAccBufs);
          q.next(kScaleSlots);
        }
        if (!ok) break;
      }
      if (T::s2q) {
        // INT4 stage 2 as r/128 more groups of the same accumulation: I * s_V[col] * s_H[row]
        if (ti.need_h) {  // the requantized H and its scales are complete
          if (!(ok = kPair ? wait_bar_cluster(hb_ready, hbq_phase, abort_flag, kSiteDrainHbq)
                           : wait_bar(hb_ready, hbq_phase, abort_flag, kSiteDrainHbq)))
            break;
          hbq_phase ^= 1u;
        }
        for (int g2 = 0; g2 < args.r / 128; ++g2) {
          const float sh = shq[row_in * 2 + g2];
          if (!(ok = wait_bar(&acc_full[a.idx], a.phase, abort_flag, kSiteDrainAccFull))) break;
          tc_fence_after();
          if (!(ok = wait_bar(&sc_full[q.idx], q.phase, abort_flag, kSiteDrainScaleFull))) break;
          drain_group(acc, tmem_base + lane_addr + a.idx * BN + c0, ncols, scl + q.idx * BN + c0,
                      sh);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&acc_empty[a.idx]);
            mbar_arrive(&sc_empty[q.idx]);
          }
          a.next(kAccBufs);
          q.next(kScaleSlots);
        }
        if (!ok) break;
      }
      // -------------------------------------------------------- epilogue
      // 16 columns at a time: stage-2 result from TMEM, plus the residual sum.
      if (T::s2) {
        if (!(ok = wait_bar(&acc_full[a.idx], a.phase, abort_flag, kSiteDrainAccFull))) break;
        tc_fence_after();
      }
#pragma unroll
      for (int j = 0; j < 64; j += 16) {
        float lr[16];
        if (T::s2) {
          uint32_t t0[8], t1[8];
          tmem_ld8(tmem_base + lane_addr + a.idx * BN + c0 + j, t0);
          tmem_ld8(tmem_base + lane_addr + a.idx * BN + c0 + j + 8, t1);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            lr[k] = __uint_as_float(t0[k]);
            lr[k + 8] = __uint_as_float(t1[k]);
          }
        }
        if (row_ok) {
          if (T::out_f32) {
            float* o = static_cast<float*>(args.out) + row * args.n + n0 + c0 + j;
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
              float4 v;
              if (T::res)
                v = make_float4(acc[j + k] * kDq, acc[j + k + 1] * kDq,
                                acc[j + k + 2] * kDq, acc[j + k + 3] * kDq);
              else
                v = make_float4(lr[k], lr[k + 1], lr[k + 2], lr[k + 3]);
              *reinterpret_cast<float4*>(o + k) = v;
            }
          } else {
            uint16_t* o = static_cast<uint16_t*>(args.out) + row * args.n + n0 + c0 + j;
            float y[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              if (T::s2)
                y[k] = acc[j + k] * kDq + lr[k];
              else
                y[k] = acc[j + k] * kDq;
            }
#pragma unroll
            for (int k = 0; k < 16; k += 8) {
              uint4 v;
              v.x = pack_bf16x2(y[k + 0], y[k + 1]);
              v.y = pack_bf16x2(y[k + 2], y[k + 3]);
              v.z = pack_bf16x2(y[k + 4], y[k + 5]);
              v.w = pack_bf16x2(y[k + 6], y[k + 7]);
              *reinterpret_cast<uint4*>(o + k) = v;
            }
          }
        }
      }
      if (T::s2) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[a.idx]);
        a.next(kAccBufs);
      }
    }
  }

  __syncthreads();
  // A CTA of a pair leaves only after its peer is done: no store or arrive from the
  // peer can still be on its way into this CTA's shared memory.
  if (kPair) cluster_sync_startup();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
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

bool encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

// Clusters of two CTAs of the pair kernel that fit on the device at once, once
// per instantiation (0 if the query fails: no pairs then).
template <int kMode, int BN, bool kA8>
int resident_pairs() {
  // Concurrent first calls may both run the query; they store the same value.
  static std::atomic<int> cached_atomic{-1};
  int cached = cached_atomic.load(std::memory_order_acquire);
  if (cached < 0) {
    using L = SmemLayout<BN, kA8>;
    auto kern = twq_gemm_kernel<kMode, BN, true, kA8>;
    int nc = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = L::kAlloc;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();  // the query's own error: pairs are simply not used
        nc = 0;
      }
    } else {
      (void)cudaGetLastError();
    }
    cached = nc > 0 ? nc : 0;
    cached_atomic.store(cached, std::memory_order_release);
  }
  return cached;
}

template <int kMode, int BN, bool kA8 = false>
cudaError_t launch_mode(const GemmCall& c, cudaStream_t st) {
  using L = SmemLayout<BN, kA8>;
  using T = ModeTraits<kMode>;
  const twq_weights* w = c.w;
  GemmArgs a{};
  a.sx = c.sx;
  a.sr = w->sr;
  a.sl1 = w->sl1;
  a.out = c.out;
  a.b = c.b;
  a.m = static_cast<int>(w->m);
  a.n = static_cast<int>(w->n);
  a.r = static_cast<int>(w->r);
  a.G = a.m / 128;
  a.row_blocks = static_cast<int>((c.b + kBM - 1) / kBM);
  a.col_tiles = T::out_h ? 1 : a.n / BN;
  // CTA pairs share H: modes with an on-chip H and stage 2, an even number of
  // column tiles, and 128 < r <= 256 in two halves of whole 16-column MMA units.
  // A step costs about the same at any MMA width up to 128, so halving H's columns
  // pays only where it halves a CTA's H steps (two 128-wide chunks become one), and
  // only where that saves more than the SMs that pairs leave idle (clusters are
  // placed within a GPC): the choice compares the K-group steps of the busiest CTA.
  bool pair = false;
  if constexpr (T::h && (T::s2 || T::s2q) && !T::h_global) {
    // (INT4 stage 2: each CTA of a pair then owns exactly one group of 128 of r)
    if (a.col_tiles % 2 == 0 && a.r % 32 == 0 && a.r > kHChunk && a.r <= 2 * kHChunk &&
        (!T::s2q || a.r == 2 * kHChunk)) {
      const int pairs = resident_pairs<kMode, BN, kA8>();
      const int hc1 = (a.r + kHChunk - 1) / kHChunk;
      const int kc = (a.r + 63) / 64;
      const int n1 = a.row_blocks * a.col_tiles, n2 = a.row_blocks * (a.col_tiles / 2);
      const double t1 = static_cast<double>(n1) / std::min(n1, num_sms());
      const double t2 = static_cast<double>(n2) / std::min(n2, pairs);
      const double s1 = t1 * (a.G + kc) + (1.0 + t1 / a.col_tiles) * hc1 * a.G;
      const double s2 = t2 * (a.G + kc) + (1.0 + t2 / (a.col_tiles / 2)) * a.G;
      pair = pairs > 0 && s2 < 0.98 * s1;
    }
  }
  a.tiles_per_rb = pair ? a.col_tiles / 2 : a.col_tiles;
  a.num_tiles = a.row_blocks * a.tiles_per_rb;
  a.r_pad = ((a.r + 63) / 64) * 64;
  a.h_box = pair ? a.r / 2 : (a.r < kHChunk ? a.r : kHChunk);

  CUtensorMap m_xq{}, m_rq{}, m_l1q{}, m_l2t{}, m_h{};
  const uint64_t kb = static_cast<uint64_t>(a.m / 2);
  // W4A8: 128 int8 codes per row and group, with the 128-byte swizzle the MMA reads
  bool ok = kA8 ? encode_2d(&m_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.xq, a.m, c.b, a.m, 128, kBM,
                            CU_TENSOR_MAP_SWIZZLE_128B)
                : encode_2d(&m_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.xq, kb, c.b, kb, 64, kBM,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
  if (T::res)
    ok = ok && encode_2d(&m_rq, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->rq, kb, a.n, kb, 64, BN,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
  if (T::h)
    ok = ok && encode_2d(&m_l1q, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->l1q, kb, a.r, kb, 64, a.h_box,
                         CU_TENSOR_MAP_SWIZZLE_NONE);
  if (T::s2)
    ok = ok && encode_2d(&m_l2t, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->l2t, a.r, a.n,
                         static_cast<uint64_t>(a.r) * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (T::s2q) {  // the 4-bit L2 codes: n rows of r/2 bytes, 64 bytes (128 codes) per group
    a.sl2q = c.sl2q;
    ok = ok && c.l2q && c.sl2q &&
         encode_2d(&m_l2t, CU_TENSOR_MAP_DATA_TYPE_UINT8, c.l2q, a.r / 2, a.n,
                   static_cast<uint64_t>(a.r / 2), 64, BN, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (T::h_global)
    ok = ok && encode_2d(&m_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c.h_global, a.r, c.b,
                         static_cast<uint64_t>(a.r) * 2, 64, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;

  if (!pair || !(T::h && (T::s2 || T::s2q) && !T::h_global)) {
    auto kern = twq_gemm_kernel<kMode, BN, false, kA8>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    int grid = a.num_tiles < num_sms() ? a.num_tiles : num_sms();
    kern<<<grid, kThreads, L::kAlloc, st>>>(m_xq, m_rq, m_l1q, m_l2t, m_h, a);
    return cudaGetLastError();
  }
  if constexpr (T::h && (T::s2 || T::s2q) && !T::h_global) {
  auto kern = twq_gemm_kernel<kMode, BN, true, kA8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1), 1, 1);
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
  // One wave of persistent pairs: as many as can be resident at once.
  const int rp = resident_pairs<kMode, BN, kA8>();
  const int pairs = a.num_tiles < rp ? a.num_tiles : rp;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
  e = cudaLaunchKernelEx(&cfg, kern, m_xq, m_rq, m_l1q, m_l2t, m_h, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
  } else {
    return cudaErrorInvalidValue;  // unreachable: `pair` implies the condition above
  }
}

}  // namespace

cudaError_t launch_gemm(const GemmCall& c, cudaStream_t st, int* launches) {
  if (c.a8 && c.mode != kModeFused && c.mode != kModeW4A4) return cudaErrorInvalidValue;
  if (launches) ++*launches;
  // Prefill batches of the three layer modes run on CTA pairs (256 x 256 tiles).
  if (pair_eligible(c)) return launch_pair(c, st);
  switch (c.mode) {
    case kModeFused:
      return c.a8 ? launch_mode<kModeFused, 128, true>(c, st) : launch_mode<kModeFused, 128>(c, st);
    case kModeW4A4:
      return c.a8 ? launch_mode<kModeW4A4, 128, true>(c, st) : launch_mode<kModeW4A4, 128>(c, st);
    case kModeLowRank: return launch_mode<kModeLowRank, 128>(c, st);
    case kModeResF32: return launch_mode<kModeResF32, 128>(c, st);
    case kModeHOnly: return launch_mode<kModeHOnly, 128>(c, st);
    case kModeS2F32: return launch_mode<kModeS2F32, 128>(c, st);
    case kModeFusedS2Q: return launch_mode<kModeFusedS2Q, 128>(c, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_and_clear_device_status(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  *code = v;
  return e;
}

}  // namespace twq
