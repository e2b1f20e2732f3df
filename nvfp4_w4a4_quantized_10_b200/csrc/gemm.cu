// Block-scaled NVFP4 x NVFP4 GEMM with a dequantizing epilogue, and the fused
// multi-segment projection, for sm_100a.
//
// What it computes [picx.dev summary of "Why Gated DeltaNet Survives 4-Bit
// Quantization", "Background": native 4-bit tensor-core GEMMs on NVFP4
// operands; anthology record LIT-800, "Standing in the anthology", and the
// cctest.ai article, "Main findings": fused projections must apply each
// module's own global scale]:
//   out[m,n] = alpha(n) * sum_b sA[m,b] sW[n,b] sum_{k in b} e2m1(A[m,k]) e2m1(W[n,k])
//   alpha(n) = 1 / (gA * gW[segment of n])
//
// Design (one persistent CTA per SM):
//   warp 0    TMA producer: per 256-wide K step, one 2-D TMA box of each
//             operand's codes (128-byte rows, 128B swizzle) and one or two
//             bulk copies of the pre-swizzled E4M3 scale chunks, all landing
//             on one mbarrier with an expected byte count.
//   warp 1    TMEM allocator and MMA issuer: per step, four tcgen05.mma
//             kind::mxf4nvf4 block_scale (K = 64 each) into the FP32
//             accumulator in TMEM, then tcgen05.commit to release the stage.
//   warps 2-5 epilogue: tcgen05.ld the accumulator (one TMEM lane per
//             output row), scale by alpha, round once to bf16 (or keep
//             f32), free the accumulator, store.  With an in-kernel
//             activation (nvfp4_linear) they first quantize X into shared
//             memory.
//   warps 6+  scale copies: one warp for P's scale chunks and one per
//             128-row block of Q's move each step's scales into TMEM
//             (tcgen05.cp 32x128b.warpx4) and signal the MMA warp.  Each
//             tcgen05 instruction holds its issuing thread for tens of
//             cycles; spread over warps, copies and MMAs overlap.
// Two tile shapes:
//   normal  P = activations (128-row tiles), Q = weight (256-row tiles):
//           prefill and fused projections.
//   swap    P = weight (128-row tiles), Q = all activation rows (<= 128):
//           decode, so the 128-row MMA dimension walks the weight; the
//           K loop is split over the CTAs (stream-K) so every SM streams W.
// Every mbarrier wait is bounded (see ptx.cuh); on timeout the CTA drains
// its in-flight copies and MMAs (bounded again), frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "block_quant.cuh"
#include "common.h"
#include "ptx.cuh"

namespace nvfp4 {

constexpr int kBM = 128;          // MMA M: rows of operand P per tile
constexpr int kSfChunk = 512;     // bytes of one 128-row x 4-scale chunk
constexpr int kTmemCols = 512;
constexpr int kGroupP = 64;       // tile raster: 64 P-tiles (8192 rows) share each Q-tile sweep
constexpr int kStageOutBytes = 16384;   // one 128-row x 128-byte output sub-tile
constexpr int kEpiBar = 1;        // named barrier id of the 128 epilogue threads

struct alignas(64) GemmParams {
  CUtensorMap tmap_p;
  CUtensorMap tmap_q;
  CUtensorMap tmap_out;  // output [M, N] in 128-byte-wide boxes (normal tiles, TMA store path)
  const uint8_t* sf_p;
  const uint8_t* sf_q;
  void* out;
  uint64_t* ws;          // swapped tiles: tagged FP32 partial tiles, 2 slots per CTA (all words empty between launches)
  unsigned* err;
  uint64_t timeout_ns;   // bound of every wait for work to arrive
  uint64_t drain_ns;     // bound of the waits for a CTA's own copies and MMAs before it exits (>= 1 s)
  int64_t M, N;          // output [M, N]
  int rows_p, rows_q;    // rows of the P and Q operands
  int rb_q;              // 128-row scale blocks allocated for Q
  int kc;                // scale chunks per row block: ceil(K / 64), MXFP4 ceil(K / 128)
  int kmma;              // ceil(K / 64): MMAs per row of tiles
  int kt;                // ceil(K / (64 * kKB)): pipeline steps per tile
  int tiles_p, tiles_q;
  int tma_store;         // 1: output through shared memory and TMA stores
  int w_static;          // 1: the weight lies in memory declared read-only (nvfp4_declare_static)
  int n_seg;
  int test_stall;        // failure-path test only: the split-tile adder never sees its helpers' partials
  int group_p;           // tile raster: P tiles per Q-tile sweep
  CUtensorMap tmap_sfa;  // CTA pairs: scale chunks of P and Q as [chunks, 128] 32-bit words
  CUtensorMap tmap_sfb;
  int seg_end[NVFP4_MAX_SEGMENTS];
  float seg_alpha[NVFP4_MAX_SEGMENTS];
  // activation quantized in the kernel (swapped tiles only): X [M, K]
  // row-major, its global scale, K
  const void* x;
  float x_gs;
  int64_t K;
  // buffer extents, checked by the debug build's bounds checks
  uint64_t sf_p_bytes, sf_q_bytes;   // scale buffers
  uint64_t out_elems;                // M * N
  uint64_t ws_words;                 // K-split workspace, 64-bit words
  uint64_t x_bytes;                  // in-kernel activation X
};

// QX: 0 = the Q operand (activations) arrives quantized, as codes and scales
// in global memory; 1 / 2 = swapped tiles whose activation X (bf16 / f32) the
// kernel quantizes itself into shared memory, all of the CTA's K-steps at
// once, before the first MMA.
// MX: MXFP4 operands (32-element blocks, E8M0 scales, kind::mxf4 with two
// scales per MMA) instead of NVFP4 (16-element blocks, E4M3 scales).
// PAIR: prefill tiles of 256 x 256 computed by a pair of CTAs (a cluster of
// two): each CTA loads its 128 activation rows and half of the 256 weight
// rows (plus all 256 rows' scales); the even CTA issues the M = 256 MMAs and
// scale copies for both (tcgen05 cta_group::2); each CTA drains its own 128
// accumulator rows.
template <int BN, bool SWAP, int QX = 0, bool MX = false, bool PAIR = false>
struct Cfg {
  static constexpr bool kQx = QX != 0;
  // K per pipeline step: kKB blocks of 64 (one MMA each), 256 deep, as
  // 128-byte rows with the 128B swizzle.  (128-deep steps with 64-byte rows
  // and the 64B swizzle also work, and fit twice as many stages, but measured
  // 40 % slower on prefill tiles: the per-step barrier and commit work then
  // outweighs the earlier buffer release.)
  static constexpr int kKB = 4;
  static constexpr int kRowBytes = 32 * kKB;                         // code bytes per row per step
  static constexpr uint32_t kSwizzleLayout = kRowBytes == 128 ? 2u : 4u;   // descriptor layout type
  static constexpr uint32_t kSbo = 8 * kRowBytes;                    // bytes between 8-row groups
  static constexpr int kSfbBlocks = (BN + 127) / 128;                // 128-row scale blocks of Q
  static constexpr int kABytes = kBM * kRowBytes;
  static constexpr int kBBytes = kQx ? 0 : (PAIR ? BN / 2 : BN) * kRowBytes;   // Q codes per stage (per CTA)
  // scale chunks (128 rows x 4 scales, 512 bytes) per step: a chunk covers 64
  // K-elements of 16-element blocks (one MMA), or 128 of 32-element blocks
  static constexpr int kChunks = MX ? kKB / 2 : kKB;
  static constexpr int kSfaBytes = kChunks * kSfChunk;
  static constexpr int kSfbBytes = kQx ? 0 : kSfbBlocks * kChunks * kSfChunk;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static constexpr int kOutBytes = SWAP ? 0 : 2 * kStageOutBytes;    // double-buffered output sub-tiles
  // in-kernel activation: codes (BN rows x 128 B, 128B swizzle) and one
  // 128-row scale block per K-step, for up to kActSteps steps
  static constexpr int kActSteps = kQx ? (BN <= 16 ? 8 : 16) : 0;
  static constexpr int kActCodeBytes = BN * kRowBytes;
  static constexpr int kActSfBytes = kKB * kSfChunk;
  static constexpr int kActBytes = kActSteps * (kActCodeBytes + kActSfBytes);
  // CTA pairs keep 4 stages although 5 fit: 5 ran 2-7 % slower on every
  // prefill and fused shape measured (the deeper ring lets the copy warps
  // run further ahead of MMAs that are not waiting on data)
  static constexpr int kMaxStages = PAIR ? 4 : 8;
  // Decode tiles with a small activation side keep to under half of the
  // SM's shared memory (and TMEM, and 128 registers), so two CTAs fit on an
  // SM.  With BN = 16 the grid has 2 x SMs CTAs: each streams half as much
  // weight and each SM keeps twice the stages in flight (decode step 12.4
  // against 13.3 us at 8x12288x5120; four stages measured 2 % faster than
  // five).  The profiler's occupancy limits are two CTAs per SM and it sees
  // about 1.8 resident on average, but the occupancy API reports one.  A
  // split tile's summing CTA waits only for partials that CTAs with higher
  // indices produce as their first work item, so the grid completes whenever
  // CTAs start in index order, resident together or not (bounded waits
  // report a timeout otherwise); the opt-in cooperative launch sizes the
  // grid to what the occupancy API admits instead.  BN = 32, and the MXFP4
  // decode tile (13.5 against 10.9 us), are slower at two per SM and keep
  // one CTA per SM.  The in-kernel activation variant follows the same grid (its
  // BN = 16 form holds 8 K-steps of activation instead of 16, covering the
  // same shapes).
  static constexpr bool kCoRes = SWAP && (kQx ? BN <= 16 : BN <= 32);
  static constexpr int kMinBlocks = kCoRes ? 2 : 1;
  static constexpr int kGridPerSm = SWAP && BN <= 16 && !MX ? 2 : 1;
  static constexpr int kSmemBudget = kCoRes ? 104 * 1024 : 222 * 1024;
  static constexpr int kFit = (kSmemBudget - kOutBytes - kActBytes) / kStageBytes;
  static constexpr int kStages = kFit < kMaxStages ? kFit : kMaxStages;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kABytes;
  static constexpr int kOffSfa = kOffB + kStages * kBBytes;
  static constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
  static constexpr int kOffAct = kOffSfb + kStages * kSfbBytes;      // 1024-aligned
  static constexpr int kOffActSf = kOffAct + kActSteps * kActCodeBytes;
  static constexpr int kOffOut = kOffActSf + kActSteps * kActSfBytes;   // 1024-aligned
  static constexpr int kOffBar = kOffOut + kOutBytes;
  // Extra warps issue the scale copies (warp 6: P's scales, warp 7 + rb: the
  // scales of Q's 128-row block rb) so that the MMA warp issues only MMAs; a
  // tcgen05 instruction holds its issuing thread for tens of cycles, but
  // instructions from different threads proceed in parallel.
  static constexpr int kCopyWarps = 1 + kSfbBlocks;
  static constexpr int kThreads = 192 + 32 * kCopyWarps;
  // full, empty, acc_full, acc_empty, drain, one scales-ready barrier per
  // stage, one drain barrier per copy warp, and (in-kernel activation) one
  // activation-ready barrier per K-step
  static constexpr int kNumBars = 2 * kStages + 3 + kStages + kCopyWarps + kActSteps;
  static constexpr int kOffSeg = kOffBar + kNumBars * 8;             // segment table: ends, alphas
  static constexpr int kOffMisc = kOffSeg + 2 * 4 * NVFP4_MAX_SEGMENTS;
  static constexpr int kOffRtab = kOffMisc + 16;                     // in-kernel activation: g / e4m3(s)
  static constexpr int kSmemBytes = kOffRtab + (kQx ? 1024 : 0) + 1024;   // + alignment slack
  // TMEM columns.  Normal 128x256 tiles: the copy warps run ahead of the
  // MMAs, so the scales of successive steps use a ring of regions at the top
  // of TMEM ([320,512) for four 48-column regions); the two accumulator
  // buffers, [0,256) and [kAcc1Col, kAcc1Col + 256), fill the rest and
  // overlap, so tile t+1 can start as soon as the epilogue has drained the
  // shared columns of tile t (it drains those 64-column slots first).
  // Swapped (decode) tiles: one accumulator and one scale region per
  // pipeline stage.
  static constexpr int kAccCols = BN < 32 ? 32 : BN;
  static constexpr bool kOverlapAcc = !SWAP && BN == 256;
  static constexpr int kSfaCols = 4 * kChunks;                       // 4 columns per chunk
  static constexpr int kSfbCols = kSfbBlocks * 4 * kChunks;
  static constexpr int kSfStageCols = kSfaCols + kSfbCols;
  // four regions (192 columns) let the copy warps run up to three steps
  // ahead; the accumulators then share 192 columns (3 slots drained first)
  static constexpr int kSfRegions = kOverlapAcc ? 4 : kStages;
  static constexpr int kSfBase = kOverlapAcc ? kTmemCols - kSfRegions * kSfStageCols : kAccCols;
  static constexpr int kAcc1Col = kOverlapAcc ? kSfBase - 256 : 0;
  static constexpr int kSharedSlots = kOverlapAcc ? (256 - kAcc1Col + 63) / 64 : 0;   // drained before release
  static constexpr int kTmemAlloc = kCoRes ? 256 : kTmemCols;         // columns this CTA allocates
  static_assert(kAcc1Col % 32 == 0, "accumulator column alignment");
  static_assert(kStages >= 2, "pipeline depth");
  static_assert(kSfBase + kSfRegions * kSfStageCols <= kTmemAlloc, "TMEM budget");
  static_assert(!kCoRes || kSmemBytes <= 113 * 1024, "under half of the SM's shared memory");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(BN % 16 == 0 && BN <= 256, "MMA N");
  static_assert(!kQx || (SWAP && BN <= 32), "in-kernel activation: swapped tiles, M <= 32");
  static_assert(!(kQx && MX), "in-kernel activation: NVFP4 only");
  static_assert(!PAIR || (!SWAP && BN == 256 && !kQx), "CTA pairs: normal 256 x 256 tiles");
  static constexpr int kMmaM = PAIR ? 2 * kBM : kBM;                 // MMA M (over the pair)
  static constexpr int kGroupTiles = PAIR ? kGroupP / 2 : kGroupP;   // raster group, in tiles of P
  static_assert(kOffAct % 1024 == 0 && kActCodeBytes % 1024 == 0, "activation tiles on swizzle atoms");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // round to nearest even
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void tile_coords(const GemmParams& p, int tile, int& tp, int& tq) {
  const int per_group = p.group_p * p.tiles_q;
  const int group = tile / per_group;
  const int first = group * p.group_p;
  const int gsize = min(p.tiles_p - first, p.group_p);
  const int local = tile - group * per_group;
  tp = first + local % gsize;
  tq = local / gsize;
}

// Work of one CTA, as a sequence of (tile, k-step range) items.
//   normal tiles: whole tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
//   swapped tiles (stream-K): the tiles_p * kt (tile, k-step) units are cut
//   into gridDim.x contiguous, balanced ranges; CTA c owns units
//   [floor(c U / G), floor((c+1) U / G)).  An item is the part of that range
//   inside one tile.
//   CTA pairs: whole 256 x 256 tiles t = pair, pair + pairs, ... for the
//   pair index blockIdx.x / 2.
struct WorkIter {
  int64_t u, u_end;   // swapped: unit range; normal: next tile index, tile count
  int kt;
  bool swap, pair;
};

__device__ __forceinline__ int64_t unit_begin(int64_t c, int64_t U, int64_t G) { return c * U / G; }

// CTA whose range holds unit u: the largest c with floor(c U / G) <= u.
__device__ __forceinline__ int64_t cta_of_unit(int64_t u, int64_t U, int64_t G) {
  return ((u + 1) * G + U - 1) / U - 1;
}

__device__ __forceinline__ WorkIter work_begin(const GemmParams& p, bool swap, bool pair = false) {
  WorkIter w;
  w.kt = p.kt;
  w.swap = swap;
  w.pair = pair;
  if (swap) {
    const int64_t U = (int64_t)p.tiles_p * p.kt, G = gridDim.x;
    w.u = unit_begin(blockIdx.x, U, G);
    w.u_end = unit_begin(blockIdx.x + 1, U, G);
  } else {
    w.u = pair ? blockIdx.x / 2 : blockIdx.x;
    w.u_end = (int64_t)p.tiles_p * p.tiles_q;
  }
  return w;
}

__device__ __forceinline__ bool work_next(const GemmParams& p, WorkIter& w, int& tp, int& tq, int& kb, int& ke) {
  if (w.u >= w.u_end) return false;
  if (w.swap) {
    tp = (int)(w.u / w.kt);
    tq = 0;
    kb = (int)(w.u - (int64_t)tp * w.kt);
    const int64_t rest = w.u_end - w.u;
    ke = (int)(kb + rest < w.kt ? kb + rest : w.kt);
    w.u += ke - kb;
  } else {
    tile_coords(p, (int)w.u, tp, tq);
    kb = 0;
    ke = w.kt;
    w.u += w.pair ? gridDim.x / 2 : gridDim.x;
  }
  return true;
}

// Segment of output column n, from the table the CTA copied to shared memory.
__device__ __forceinline__ int seg_index_smem(const int* ends, int n_seg, int64_t n) {
  int i = 0;
  while (i < n_seg - 1 && n >= ends[i]) ++i;
  return i;
}

__device__ __forceinline__ float seg_alpha_smem(const int* ends, const float* alphas, int n_seg, int64_t n) {
  return alphas[seg_index_smem(ends, n_seg, n)];
}

// Tagged partial words: FP32 bits in the low half, kFullTag in the high half
// once written; 0 = empty.  An aligned 64-bit store or load is single-copy
// atomic, so a reader that sees the tag sees the value.
constexpr uint32_t kFullTag = 1u;

__device__ __forceinline__ void st_full_word(uint64_t* p, uint32_t value_bits) {
  const uint64_t w = ((uint64_t)kFullTag << 32) | value_bits;
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

__device__ __forceinline__ void st_word(uint64_t* p, uint64_t w) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

// No "memory" clobber: the polls of one round are independent and may all be
// in flight together (volatile keeps each round's loads inside its loop).
__device__ __forceinline__ uint64_t ld_word(const uint64_t* p) {
  uint64_t w;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(p));
  return w;
}

// Byte offset of 16-byte chunk c of row r in a 128-row x 128-byte sub-tile
// stored with the 128B swizzle the output tensor map uses.
__device__ __forceinline__ uint32_t swz128(uint32_t r, uint32_t c) { return r * 128 + ((c ^ (r & 7)) << 4); }

template <int BN, bool SWAP, bool OUT_F32, int QX = 0, bool MX = false, bool PAIR = false>
__global__ void __launch_bounds__(Cfg<BN, SWAP, QX, MX, PAIR>::kThreads, Cfg<BN, SWAP, QX, MX, PAIR>::kMinBlocks)
    nvfp4_gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<BN, SWAP, QX, MX, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + C::kOffBar;
  const uint32_t bar_empty = bar_full + 8 * C::kStages;
  const uint32_t bar_acc_full = bar_empty + 8 * C::kStages;
  const uint32_t bar_acc_empty = bar_acc_full + 8;
  const uint32_t bar_drain = bar_acc_empty + 8;
  const uint32_t bar_sf = bar_drain + 8;                     // [kStages]
  const uint32_t bar_cp_drain = bar_sf + 8 * C::kStages;     // [kCopyWarps]
  const uint32_t bar_act = bar_cp_drain + 8 * C::kCopyWarps;  // [kActSteps] in-kernel activation ready
  int* seg_end_s = reinterpret_cast<int*>(smem + C::kOffSeg);
  float* seg_alpha_s = reinterpret_cast<float*>(smem + C::kOffSeg + 4 * NVFP4_MAX_SEGMENTS);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pairs: rank in the pair; the even CTA (leader) issues the tcgen05 work
  const uint32_t prank = PAIR ? (cluster_ctarank() & 1u) : 0u;
  const bool leader = prank == 0;
  // the next kernel in the stream may launch now; it waits for this grid's
  // completion before touching anything this grid reads or writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    mbar_init(bar_acc_full, 1);
    // CTA pairs: one arrival per epilogue warp of either CTA; otherwise one
    // per epilogue thread
    mbar_init(bar_acc_empty, PAIR ? 8 : 128);
    mbar_init(bar_drain, 1);
    for (int s = 0; s < C::kStages; ++s) mbar_init(bar_sf + 8 * s, C::kCopyWarps);
    for (int i = 0; i < C::kCopyWarps; ++i) mbar_init(bar_cp_drain + 8 * i, 1);
    for (int j = 0; j < C::kActSteps; ++j) mbar_init(bar_act + 8 * j, 128);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&p.tmap_p);
    prefetch_tmap(&p.tmap_q);
    if (!SWAP && p.tma_store) prefetch_tmap(&p.tmap_out);
    if (PAIR) {
      prefetch_tmap(&p.tmap_sfa);
      prefetch_tmap(&p.tmap_sfb);
    }
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + NVFP4_MAX_SEGMENTS) {
    seg_end_s[threadIdx.x - 64] = p.seg_end[threadIdx.x - 64];
    seg_alpha_s[threadIdx.x - 64] = p.seg_alpha[threadIdx.x - 64];
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      // both CTAs of the pair allocate together (the same columns in each)
      tmem_alloc_pair(smem_u32(tmem_holder), C::kTmemAlloc);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_holder), C::kTmemAlloc);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the even CTA's barriers are initialised before the odd CTA of its pair
  // can arrive on them
  if constexpr (PAIR) cluster_sync();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Programmatic dependent launch: this kernel may start while the
    // preceding kernel in the stream still runs, and that kernel may be
    // writing any of the inputs (the weight included).  Before
    // griddepcontrol.wait the weight tiles of the first kStages steps are
    // only prefetched into L2 (a hint that reads nothing into the CTA); every
    // load into shared memory comes after the wait.
    if (lane == 0) {
      const int kc = p.kc, rb_q = p.rb_q;
      uint32_t issued_mask = 0, last_parity = 0;   // for the drain on abort
      bool ok = true;
      // p0: this CTA's first row of P (CTA pairs: its 128-row half of the
      // 256-row tile); q0: the tile's first row of Q
      auto for_steps = [&](WorkIter w, int first, int count, auto&& fn) {
        int tp, tq, kb, ke, j = 0;
        while (j < first + count && work_next(p, w, tp, tq, kb, ke))
          for (int k = kb; k < ke && j < first + count; ++k, ++j)
            if (j >= first) fn(j, PAIR ? tp * 2 * kBM + (int)prank * kBM : tp * kBM, tq * BN, k);
      };
      auto nsfb_of = [&](int q0) {
        int n = 0;
#pragma unroll
        for (int rb = 0; rb < C::kSfbBlocks; ++rb)
          if ((q0 >> 7) + rb < rb_q) ++n;
        return n;
      };
      auto load_p = [&](int stage, int p0, int k) {
        const uint32_t fb = bar_full + 8 * stage;
        const int nch = min(C::kChunks, kc - C::kChunks * k);
        if constexpr (PAIR) {
          // into this CTA's shared memory, completing on the even CTA's barrier
          tma_load_2d_pair(sbase + C::kOffA + stage * C::kABytes, &p.tmap_p, k * C::kRowBytes, p0, fb);
          tma_load_2d_pair(sbase + C::kOffSfa + stage * C::kSfaBytes, &p.tmap_sfa, 0, (p0 >> 7) * kc + C::kChunks * k,
                           fb);
          return;
        }
        tma_load_2d(sbase + C::kOffA + stage * C::kABytes, &p.tmap_p, k * C::kRowBytes, p0, fb);
        size_t off = ((size_t)(p0 >> 7) * kc + C::kChunks * k) * kSfChunk;
        if (!bounds_ok(off + (size_t)nch * kSfChunk <= p.sf_p_bytes, p.err)) off = 0;
        bulk_load(sbase + C::kOffSfa + stage * C::kSfaBytes, p.sf_p + off, (uint32_t)nch * kSfChunk, fb);
      };
      auto load_q = [&](int stage, int q0, int k) {
        const uint32_t fb = bar_full + 8 * stage;
        if constexpr (PAIR) {
          // this CTA's 128-row half of the weight tile, and the scales of all
          // 256 rows (both CTAs copy them into their own TMEM)
          tma_load_2d_pair(sbase + C::kOffB + stage * C::kBBytes, &p.tmap_q, k * C::kRowBytes, q0 + (int)prank * kBM,
                           fb);
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
            tma_load_2d_pair(sbase + C::kOffSfb + stage * C::kSfbBytes + rb * C::kChunks * kSfChunk, &p.tmap_sfb, 0,
                             ((q0 >> 7) + rb) * kc + C::kChunks * k, fb);
          return;
        }
        const uint32_t sf_bytes = (uint32_t)min(C::kChunks, kc - C::kChunks * k) * kSfChunk;
        const int nsfb = nsfb_of(q0);
        tma_load_2d(sbase + C::kOffB + stage * C::kBBytes, &p.tmap_q, k * C::kRowBytes, q0, fb);
#pragma unroll
        for (int rb = 0; rb < C::kSfbBlocks; ++rb)
          if (rb < nsfb) {
            size_t off = ((size_t)((q0 >> 7) + rb) * kc + C::kChunks * k) * kSfChunk;
            if (!bounds_ok(off + sf_bytes <= p.sf_q_bytes, p.err)) off = 0;
            bulk_load(sbase + C::kOffSfb + stage * C::kSfbBytes + rb * C::kChunks * kSfChunk, p.sf_q + off, sf_bytes,
                      fb);
          }
      };
      auto expect = [&](int stage, int q0, int k) {
        if constexpr (PAIR) {
          // the even CTA's barrier counts both CTAs' bytes (every box moves
          // its full size; rows past the tensor are zero-filled)
          if (leader)
            mbar_arrive_expect_tx(bar_full + 8 * stage,
                                  2 * (C::kABytes + C::kBBytes + C::kSfaBytes + C::kSfbBytes));
          return;
        }
        const int nch = min(C::kChunks, kc - C::kChunks * k);
        const uint32_t sf_bytes = (uint32_t)nch * kSfChunk;
        mbar_arrive_expect_tx(bar_full + 8 * stage,
                              C::kABytes + C::kBBytes + sf_bytes * (1 + (C::kQx ? 0 : nsfb_of(q0))));
      };
      const WorkIter w0 = work_begin(p, SWAP, PAIR);
      // prologue: the first kStages stages are free
      int npro = 0;
      const bool w_static = p.w_static != 0;
      for_steps(w0, 0, C::kStages, [&](int j, int p0, int q0, int k) {
        if (w_static) {
          // a weight declared read-only cannot be written by the preceding
          // kernel: load its first stages now
          expect(j, q0, k);
          if (SWAP) load_p(j, p0, k);
          else load_q(j, q0, k);
          issued_mask |= 1u << j;
        } else {
          const uint32_t sf_bytes = (uint32_t)min(C::kChunks, kc - C::kChunks * k) * kSfChunk;
          if (SWAP) {
            tma_prefetch_l2_2d(&p.tmap_p, k * C::kRowBytes, p0);
            const size_t off = ((size_t)(p0 >> 7) * kc + C::kChunks * k) * kSfChunk;
            if (bounds_ok(off + sf_bytes <= p.sf_p_bytes, p.err)) bulk_prefetch_l2(p.sf_p + off, sf_bytes);
          } else {
            tma_prefetch_l2_2d(&p.tmap_q, k * C::kRowBytes, PAIR ? q0 + (int)prank * kBM : q0);
          }
        }
        npro = j + 1;
      });
      if (SWAP) {
        // decode tiles stream each weight byte once: bring the rest of this
        // CTA's weight range into L2 now, so that HBM keeps streaming while
        // the preceding kernel finishes (a hint: it reads nothing into the CTA)
        for_steps(w0, C::kStages, 1 << 30, [&](int, int p0, int, int k) {
          const uint32_t sf_bytes = (uint32_t)min(C::kChunks, kc - C::kChunks * k) * kSfChunk;
          tma_prefetch_l2_2d(&p.tmap_p, k * C::kRowBytes, p0);
          const size_t off = ((size_t)(p0 >> 7) * kc + C::kChunks * k) * kSfChunk;
          if (bounds_ok(off + sf_bytes <= p.sf_p_bytes, p.err)) bulk_prefetch_l2(p.sf_p + off, sf_bytes);
        });
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for_steps(w0, 0, npro, [&](int j, int p0, int q0, int k) {
        if (w_static) {
          if (SWAP) {
            if (!C::kQx) load_q(j, q0, k);
          } else {
            load_p(j, p0, k);
          }
        } else {
          expect(j, q0, k);
          load_p(j, p0, k);
          if (!C::kQx) load_q(j, q0, k);
          issued_mask |= 1u << j;
        }
      });
      int stage = npro % C::kStages;
      uint32_t phase = npro == C::kStages ? 1u : 0u;
      if (npro == C::kStages) {
        for_steps(w0, npro, 1 << 30, [&](int j, int p0, int q0, int k) {
          if (!ok) return;
          if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, p.err, p.timeout_ns)) { ok = false; return; }
          expect(stage, q0, k);
          load_p(stage, p0, k);
          if (!C::kQx) load_q(stage, q0, k);
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        });
      }
      // let every issued copy land before the CTA exits, whichever role may
      // have given up (when nothing did, the last load of each stage has
      // already landed and each wait returns at once).  The odd CTA of a
      // pair cannot see its loads complete (they count on the even CTA's
      // barrier): it waits until the MMAs have consumed each stage instead,
      // and the cluster-wide barrier before exit keeps it until the even CTA
      // has drained.
      for (int s = 0; s < C::kStages; ++s)
        if (issued_mask & (1u << s)) {
          volatile int never = 0;
          if (leader) (void)mbar_wait(bar_full + 8 * s, (last_parity >> s) & 1, &never, p.err, p.drain_ns);
          else (void)mbar_wait(bar_empty + 8 * s, (last_parity >> s) & 1, &never, p.err, p.drain_ns);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp follows the pipeline; lane 0 issues every MMA.  The copy
    // warps waited for each stage's data and moved its scales into TMEM.
    constexpr uint32_t idesc = MX ? idesc_mxf4(C::kMmaM, BN) : idesc_nvf4(C::kMmaM, BN);
    // Descriptors of stage 0, k-block 0; later stages and k-blocks only move
    // the 14-bit start-address field (address >> 4), which never carries.
    const uint64_t a_desc0 = smem_desc(sbase + C::kOffA, 16, C::kSbo, C::kSwizzleLayout);
    const uint64_t b_desc0 = smem_desc(sbase + (C::kQx ? C::kOffAct : C::kOffB), 16, C::kSbo, C::kSwizzleLayout);
    const uint32_t sf_t0 = tmem_base + C::kSfBase;
    int stage = 0, region = 0, lstep = 0;    // lstep: steps of this CTA so far
    uint32_t phase = 0, acc_phase = 0, acc_buf = 0;
    bool ok = true;
    WorkIter w = work_begin(p, SWAP, PAIR);
    int tp, tq, kb0, ke0;
    // CTA pairs: only the even CTA issues (for both)
    while (ok && leader && work_next(p, w, tp, tq, kb0, ke0)) {
      if (!mbar_wait(bar_acc_empty, acc_phase ^ 1, abort_flag, p.err, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t acc = tmem_base + (acc_buf ? C::kAcc1Col : 0);
      for (int k = kb0; k < ke0; ++k) {
        if (C::kQx && lstep >= C::kActSteps) {     // the host sizes the grid so this cannot happen
          atomicCAS(p.err, 0u, kErrBounds);
          *abort_flag = 1;
          ok = false;
          break;
        }
        if (!mbar_wait(bar_sf + 8 * stage, phase, abort_flag, p.err, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t sfa_t = sf_t0 + region * C::kSfStageCols;
          const uint32_t sfb_t = sfa_t + C::kSfaCols;
          const uint64_t ad = a_desc0 + (uint64_t)((stage * C::kABytes) >> 4);
          const uint64_t bd = b_desc0 + (uint64_t)(((C::kQx ? lstep * C::kActCodeBytes : stage * C::kBBytes)) >> 4);
          const uint32_t acc_in = k != kb0 ? 1u : 0u;
          // MMA kb reads chunk kb (NVFP4, 4 scales each) or half of chunk
          // kb / 2 (MXFP4: scale bytes 0-1 or 2-3 of each TMEM column,
          // selected by the descriptor's scale-factor ids)
          const int nkb = min(C::kKB, p.kmma - C::kKB * k);
          auto mma = [&](int kb) {
            const int c = MX ? kb >> 1 : kb;
            const uint32_t id = MX ? (uint32_t)(kb & 1) * 2u : 0u;
            if constexpr (PAIR)
              tc_mma_block_scaled_pair<MX>(acc, ad + (uint64_t)(kb * 2), bd + (uint64_t)(kb * 2),
                                           idesc | (id << 29) | (id << 4), sfa_t + c * 4,
                                           sfb_t + c * 4 * C::kSfbBlocks, (acc_in | kb) != 0 ? 1u : 0u);
            else
              tc_mma_block_scaled<MX>(acc, ad + (uint64_t)(kb * 2), bd + (uint64_t)(kb * 2),
                                      idesc | (id << 29) | (id << 4), sfa_t + c * 4, sfb_t + c * 4 * C::kSfbBlocks,
                                      (acc_in | kb) != 0 ? 1u : 0u);
          };
          if (nkb == C::kKB) {
#pragma unroll
            for (int kb = 0; kb < C::kKB; ++kb) mma(kb);
          } else {
            for (int kb = 0; kb < nkb; ++kb) mma(kb);
          }
          // the stage is free in both CTAs of a pair
          if constexpr (PAIR) tc_commit_pair_both(bar_empty + 8 * stage);
          else tc_commit(bar_empty + 8 * stage);
        }
        __syncwarp();
        if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        if (++region == C::kSfRegions) region = 0;
        ++lstep;
      }
      if (!ok) break;
      if (lane == 0) {
        if constexpr (PAIR) tc_commit_pair_both(bar_acc_full);
        else tc_commit(bar_acc_full);
      }
      __syncwarp();
      acc_phase ^= 1;
      acc_buf ^= 1;
    }
    if (lane == 0 && leader) {
      // every MMA and scale copy issued by this thread has completed once
      // this commit arrives
      if constexpr (PAIR) tc_commit_pair(bar_drain);
      else tc_commit(bar_drain);
      volatile int never = 0;
      (void)mbar_wait(bar_drain, 0, &never, p.err, p.drain_ns);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int sp = warp & 3;                 // TMEM subpartition of this warp
    const int row = sp * 32 + lane;          // accumulator lane = tile row of P
    const int et = threadIdx.x - 64;         // epilogue thread index 0..127
    const uint32_t taddr = tmem_base + ((uint32_t)(sp * 32) << 16);
    const int64_t M = p.M, N = p.N;
    const int n_seg = p.n_seg;
    const bool tma_store = !SWAP && p.tma_store;
    uint32_t acc_phase = 0, acc_buf = 0;
    uint32_t out_buf = 0;                    // next staging buffer (TMA store path)
    WorkIter w = work_begin(p, SWAP, PAIR);
    const int64_t U = (int64_t)p.tiles_p * p.kt, G = gridDim.x;
    int tp, tq, kb0, ke0;
    bool first_item = true;
    if constexpr (C::kQx) {
      // ---------------------------------------------- in-kernel activation
      // Quantize the rows of X for every K-step this CTA computes, with the
      // same per-block arithmetic as the quantize kernel, into the MMA's
      // operand layout: codes of step j at kOffAct + j * BN * 128 (row m at
      // m * 128, 16-byte chunks 128B-swizzled), scales of step j at
      // kOffActSf + j * 2048 (the 512-byte chunk of K-block kb holds row m's
      // four scales at m * 16).  Rows [M, BN) and K past the end stay zero.
      constexpr bool kF32 = QX == 2;
      constexpr int kEsz = kF32 ? 4 : 2;
      // the K-steps of this CTA, in the order every role walks them
      int ks[C::kActSteps];
      int nsteps = 0;
      {
        WorkIter wq = work_begin(p, SWAP, PAIR);
        int a, b2, c0, c1;
        while (work_next(p, wq, a, b2, c0, c1))
          for (int k = c0; k < c1 && nsteps < C::kActSteps; ++k) ks[nsteps++] = k;
      }
      const int64_t K = p.K;
      const uint8_t* xb = reinterpret_cast<const uint8_t*>(p.x);
      // A thread owns (row, block) pairs et, et + 128, ... (one pair when
      // M <= 8) and handles them one after the other.  Per pair, windows of
      // kWin steps: the next window's loads are in flight while the current
      // one is quantized (all its blocks together, for instruction-level
      // parallelism: four warps alone cannot hide latency by switching).  A
      // thread publishes step j (its barrier, 128 arrivals) after its last
      // pair's block of step j is stored, so the MMAs can start early.
      // Two-step windows: the first MMAs wait for less quantizing (decode
      // step 12.7 us against 13.2 with four-step windows, 12.8 with one)
      constexpr int kWin = 2;
      const int npairs = (int)M * 16;
      const int nq = et < npairs ? (npairs - 1 - et) / 128 + 1 : 0;   // pairs of this thread
      asm volatile("griddepcontrol.wait;" ::: "memory");      // X is written by the previous kernel
      auto load_window = [&](int pair, int j0, Block16<kF32> (&B)[kWin]) {
        const int m = pair >> 4, bq = pair & 15;
#pragma unroll
        for (int u = 0; u < kWin; ++u) {
          const int jj = j0 + u;
          const int64_t e = (int64_t)(jj < nsteps ? ks[jj] : 0) * 256 + bq * 16;
          if (jj < nsteps && e < K) {
            if (bounds_ok((uint64_t)((int64_t)m * K + e + 16) * kEsz <= p.x_bytes, p.err))
              load_block_at<kF32>(xb + ((int64_t)m * K + e) * kEsz, B[u]);
            else
              B[u] = Block16<kF32>{};
          }
        }
      };
      Block16<kF32> Bc[kWin], Bn[kWin];
      if (nq > 0) load_window(et, 0, Bc);
      float* rtab = reinterpret_cast<float*>(smem + C::kOffRtab);
      rtab[et] = recip_entry(p.x_gs, (uint32_t)et);
      rtab[et + 128] = recip_entry(p.x_gs, (uint32_t)et + 128);
      for (int i = et; i < C::kActBytes / 16; i += 128)
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(sbase + C::kOffAct + 16 * i), "r"(0) : "memory");
      named_bar_sync(kEpiBar, 128);                // zeros and rtab are in place
      if (nq == 0)
        for (int jj = 0; jj < nsteps; ++jj) mbar_arrive(bar_act + 8 * jj);
      for (int q = 0; q < nq; ++q) {
        const int pair = et + 128 * q;
        const int m = pair >> 4, bq = pair & 15;
        const bool last = q == nq - 1;
        for (int j0 = 0; j0 < nsteps; j0 += kWin) {
          // prefetch: the next window of this pair, or the first of the next pair
          if (j0 + kWin < nsteps) load_window(pair, j0 + kWin, Bn);
          else if (!last) load_window(pair + 128, 0, Bn);
#pragma unroll
          for (int u = 0; u < kWin; ++u) {
            const int jj = j0 + u;
            const int64_t e = (int64_t)(jj < nsteps ? ks[jj] : 0) * 256 + bq * 16;
            if (jj < nsteps && e < K) {
              uint32_t lo, hi;
              const uint32_t sc = quantize_block<kF32>(Bc[u], p.x_gs, rtab, lo, hi);
              // byte bq * 8 of row m: 16-byte chunk bq / 2, swizzled with m % 8
              *reinterpret_cast<uint2*>(smem + C::kOffAct + jj * C::kActCodeBytes + m * 128 +
                                        ((((bq >> 1) ^ (m & 7))) << 4) + (bq & 1) * 8) = make_uint2(lo, hi);
              smem[C::kOffActSf + jj * C::kActSfBytes + (bq >> 2) * kSfChunk + m * 16 + (bq & 3)] = (uint8_t)sc;
            }
          }
          if (last) {
            fence_proxy_async_smem();              // generic-proxy writes -> tcgen05 reads
#pragma unroll
            for (int u = 0; u < kWin; ++u)
              if (j0 + u < nsteps) mbar_arrive(bar_act + 8 * (j0 + u));
          }
#pragma unroll
          for (int u = 0; u < kWin; ++u) Bc[u] = Bn[u];
        }
      }
    }
    // hand the accumulator back to the MMA warp (CTA pairs: to the even
    // CTA's MMA warp, one arrival per warp of either CTA)
    auto release_acc = [&]() {
      tc_fence_before();
      if constexpr (PAIR) {
        __syncwarp();
        if (lane == 0) {
          if (leader) mbar_arrive(bar_acc_empty);
          else mbar_arrive_cluster(map_to_rank(bar_acc_empty, 0));
        }
      } else {
        mbar_arrive(bar_acc_empty);
      }
    };
    while (work_next(p, w, tp, tq, kb0, ke0)) {
      // CTA pairs: this CTA's rows are its 128-row half of the 256-row tile
      const int64_t p0 = PAIR ? (int64_t)tp * 2 * kBM + (int64_t)prank * kBM : (int64_t)tp * kBM;
      const int64_t q0 = (int64_t)tq * BN;
      if (!mbar_wait(bar_acc_full, acc_phase, abort_flag, p.err, p.timeout_ns)) break;
      __syncwarp();
      tc_fence_after();
      if constexpr (!SWAP) {
        const int64_t m = p0 + row;
        // 64-column slots are drained starting with the columns this buffer
        // shares with the other one; TMEM is handed back right after them.
        const uint32_t tacc = taddr + (acc_buf ? C::kAcc1Col : 0);
        auto slot_col = [&](int slot) -> int {
          return C::kOverlapAcc && acc_buf == 0 ? ((slot + 4 - C::kSharedSlots) & 3) * 64 : slot * 64;
        };
        if constexpr (!OUT_F32) {
          // drain the whole accumulator row into registers (bf16 pairs)
          uint32_t packed[BN / 2];
#pragma unroll
          for (int slot = 0; slot < BN / 64; ++slot) {
            const int col = slot_col(slot);
            uint32_t r0[32], r1[32];
            tmem_ld_32x32b_x32(tacc + col, r0);
            tmem_ld_32x32b_x32(tacc + col + 32, r1);
            tmem_ld_wait();
            if (slot == C::kSharedSlots - 1 && C::kOverlapAcc) release_acc();
            const int64_t n0 = q0 + col;
            // one scale for the whole 64-column slot unless a segment
            // boundary falls inside it
            int seg_lo = 0, seg_hi = 0;
            if (n_seg > 1) {
              seg_lo = seg_index_smem(seg_end_s, n_seg, n0);
              seg_hi = seg_index_smem(seg_end_s, n_seg, n0 + 63 < N ? n0 + 63 : N - 1);
            }
            if (seg_lo == seg_hi) {
              const float a = seg_alpha_s[seg_lo];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                packed[slot * 32 + i] = pack_bf16x2(__fmul_rn(__uint_as_float(r0[2 * i]), a),
                                                    __fmul_rn(__uint_as_float(r0[2 * i + 1]), a));
                packed[slot * 32 + 16 + i] = pack_bf16x2(__fmul_rn(__uint_as_float(r1[2 * i]), a),
                                                         __fmul_rn(__uint_as_float(r1[2 * i + 1]), a));
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                packed[slot * 32 + i] =
                    pack_bf16x2(__fmul_rn(__uint_as_float(r0[2 * i]),
                                          seg_alpha_smem(seg_end_s, seg_alpha_s, n_seg, n0 + 2 * i)),
                                __fmul_rn(__uint_as_float(r0[2 * i + 1]),
                                          seg_alpha_smem(seg_end_s, seg_alpha_s, n_seg, n0 + 2 * i + 1)));
                packed[slot * 32 + 16 + i] =
                    pack_bf16x2(__fmul_rn(__uint_as_float(r1[2 * i]),
                                          seg_alpha_smem(seg_end_s, seg_alpha_s, n_seg, n0 + 32 + 2 * i)),
                                __fmul_rn(__uint_as_float(r1[2 * i + 1]),
                                          seg_alpha_smem(seg_end_s, seg_alpha_s, n_seg, n0 + 33 + 2 * i)));
              }
            }
          }
          if (!C::kOverlapAcc) release_acc();
          if (tma_store) {
            // 64-column sub-tiles through two 16 KB swizzled staging buffers
#pragma unroll
            for (int sub = 0; sub < BN / 64; ++sub) {
              // sub-tiles wholly past N are skipped outright (uniform across
              // the epilogue), so every buffer written is one whose last
              // store has been committed and waited for
              const int col = slot_col(sub);
              if (q0 + col >= N) continue;
              const uint32_t buf = sbase + C::kOffOut + out_buf * kStageOutBytes;
              if (et == 0) bulk_wait_group_read<1>();          // the store that used buf has read it
              named_bar_sync(kEpiBar, 128);
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const uint32_t* v = &packed[sub * 32 + c * 4];
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + swz128(row, c)), "r"(v[0]),
                             "r"(v[1]), "r"(v[2]), "r"(v[3])
                             : "memory");
              }
              fence_proxy_async_smem();
              named_bar_sync(kEpiBar, 128);
              if (et == 0) {
                tma_store_2d(&p.tmap_out, buf, (int32_t)(q0 + col), (int32_t)p0);
                bulk_commit_group();
              }
              out_buf ^= 1;
            }
          } else if (m < M) {
            __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + m * N;
#pragma unroll
            for (int c = 0; c < BN / 8; ++c) {
              const int64_t n = q0 + slot_col(c / 8) + (c % 8) * 8;
#pragma unroll
              for (int e = 0; e < 8; ++e)
                if (n + e < N && bounds_ok((uint64_t)(m * N + n + e) < p.out_elems, p.err))
                  reinterpret_cast<uint16_t*>(orow)[n + e] = (uint16_t)(packed[4 * c + e / 2] >> (16 * (e & 1)));
            }
          }
        } else {
          // FP32 output: 32-column chunks in slot order; TMEM is released once
          // the shared columns (the first slot) are out
#pragma unroll 1
          for (int cc = 0; cc < BN / 32; ++cc) {
            const int c = slot_col(cc / 2) / 32 + (cc & 1);
            uint32_t r[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tacc + c * 32, r);
            tmem_ld_wait();
            if (cc == 2 * C::kSharedSlots - 1 && C::kOverlapAcc) release_acc();
            const int64_t n0 = q0 + c * 32;
            int seg_lo = 0, seg_hi = 0;
            if (n_seg > 1) {
              seg_lo = seg_index_smem(seg_end_s, n_seg, n0);
              seg_hi = seg_index_smem(seg_end_s, n_seg, n0 + 31 < N ? n0 + 31 : N - 1);
            }
            if (seg_lo == seg_hi) {
              const float a = seg_alpha_s[seg_lo];
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__fmul_rn(__uint_as_float(r[i]), a));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                r[i] = __float_as_uint(
                    __fmul_rn(__uint_as_float(r[i]), seg_alpha_smem(seg_end_s, seg_alpha_s, n_seg, n0 + i)));
            }
            if (tma_store && q0 + c * 32 < N) {
              const uint32_t buf = sbase + C::kOffOut + out_buf * kStageOutBytes;
              if (et == 0) bulk_wait_group_read<1>();
              named_bar_sync(kEpiBar, 128);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + swz128(row, j)),
                             "r"(r[4 * j]), "r"(r[4 * j + 1]), "r"(r[4 * j + 2]), "r"(r[4 * j + 3])
                             : "memory");
              fence_proxy_async_smem();
              named_bar_sync(kEpiBar, 128);
              if (et == 0) {
                tma_store_2d(&p.tmap_out, buf, (int32_t)(q0 + c * 32), (int32_t)p0);
                bulk_commit_group();
              }
              out_buf ^= 1;
            } else if (!tma_store && m < M) {
              float* orow = reinterpret_cast<float*>(p.out) + m * N;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int64_t n = q0 + c * 32 + i;
                if (n < N && bounds_ok((uint64_t)(m * N + n) < p.out_elems, p.err)) orow[n] = __uint_as_float(r[i]);
              }
            }
          }
          if (!C::kOverlapAcc) release_acc();
        }
      } else {
        // swap: lane = weight row = output column n; accumulator column =
        // activation row.  The whole accumulator row goes to registers, then
        // TMEM is handed back.
        const int64_t n = p0 + row;
        const float alpha = seg_alpha_smem(seg_end_s, seg_alpha_s, n_seg, n);
        constexpr int kCols = BN < 32 ? BN : 32;
        uint32_t r[(BN + 31) / 32][kCols];
#pragma unroll
        for (int c = 0; c < (BN + 31) / 32; ++c) {
          if constexpr (BN >= 32) {
            tmem_ld_32x32b_x32(taddr + c * 32, r[c]);
          } else {
            uint32_t r8[8];
#pragma unroll
            for (int j = 0; j < BN / 8; ++j) {
              tmem_ld_32x32b_x8(taddr + j * 8, r8);
#pragma unroll
              for (int i = 0; i < 8; ++i) r[0][j * 8 + i] = r8[i];
            }
          }
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(bar_acc_empty);
        auto store_out = [&](int64_t mm, float v) {
          if (!bounds_ok((uint64_t)(mm * N + n) < p.out_elems, p.err)) return;
          if constexpr (OUT_F32) reinterpret_cast<float*>(p.out)[mm * N + n] = v;
          else reinterpret_cast<__nv_bfloat16*>(p.out)[mm * N + n] = __float2bfloat16_rn(v);
        };
        const int64_t tile_u0 = (int64_t)tp * p.kt;
        const int64_t c_first = cta_of_unit(tile_u0, U, G);
        const int64_t c_last = cta_of_unit(tile_u0 + p.kt - 1, U, G);
        if (c_first == c_last) {
          // the whole K range of this tile ran here
          if (n < N) {
#pragma unroll
            for (int c = 0; c < (BN + 31) / 32; ++c)
#pragma unroll
              for (int i = 0; i < kCols; ++i) {
                const int64_t mm = q0 + c * 32 + i;
                if (mm < M) store_out(mm, __fmul_rn(__uint_as_float(r[c][i]), alpha));
              }
          }
        } else {
          // split tile.  The CTA that holds the tile's first K steps (its last
          // work item, so it finishes last) adds the tile up in CTA (= K)
          // order, its own partial from registers.  Every other contributor
          // writes its partial to its slot (2c for CTA c's first item, 2c + 1
          // for its last) as 64-bit words that carry the FP32 value in the low
          // half and a "full" tag in the high half: one single-copy-atomic
          // store per value, so no fence or counter is needed.  The adder
          // polls each word until it is full and clears it for the next
          // launch.
          if ((int64_t)blockIdx.x != c_first) {
            const int64_t part0 = (2 * (int64_t)blockIdx.x + (first_item ? 0 : 1)) * BN * kBM + row;
            uint64_t* part = p.ws + part0;
#pragma unroll
            for (int c = 0; c < (BN + 31) / 32; ++c)
#pragma unroll
              for (int i = 0; i < kCols; ++i) {
                const int mm = c * 32 + i;
                if (q0 + mm < M && bounds_ok((uint64_t)(part0 + (int64_t)mm * kBM) < p.ws_words, p.err))
                  st_full_word(part + (int64_t)mm * kBM, r[c][i]);
              }
          } else {
            float sum[(BN + 31) / 32][kCols];
#pragma unroll
            for (int cb = 0; cb < (BN + 31) / 32; ++cb)
#pragma unroll
              for (int i = 0; i < kCols; ++i) sum[cb][i] = __uint_as_float(r[cb][i]);
            bool ok_all = true;
            for (int64_t c = c_first + 1; c <= c_last && ok_all; ++c) {
              const int64_t slot = 2 * c + (unit_begin(c, U, G) >= tile_u0 ? 0 : 1);
              // the slot's last word is inside the workspace (debug build)
              if (!bounds_ok((uint64_t)((slot + 1) * BN * kBM) <= p.ws_words, p.err)) {
                ok_all = false;
                break;
              }
              uint64_t* src = p.ws + slot * BN * kBM + row;
              // one round polls every word of a 32-column chunk at once
#pragma unroll
              for (int cb = 0; cb < (BN + 31) / 32; ++cb) {
                uint64_t v[kCols];
                const uint64_t t0 = globaltimer_ns();
                while (true) {
#pragma unroll
                  for (int i = 0; i < kCols; ++i) {
                    const int mm = cb * 32 + i;
                    v[i] = q0 + mm < M ? ld_word(src + (int64_t)mm * kBM) : (uint64_t)kFullTag << 32;
                  }
                  uint32_t all = p.test_stall ? 0u : 1u;
#pragma unroll
                  for (int i = 0; i < kCols; ++i) all &= (uint32_t)((v[i] >> 32) == kFullTag);
                  if (all) break;
                  if (globaltimer_ns() - t0 > p.timeout_ns) {
                    atomicCAS(p.err, 0u, kErrTimeout);
                    ok_all = false;
                    break;
                  }
                }
                if (!ok_all) break;
#pragma unroll
                for (int i = 0; i < kCols; ++i) {
                  const int mm = cb * 32 + i;
                  sum[cb][i] = __fadd_rn(sum[cb][i], __uint_as_float((uint32_t)v[i]));
                  if (q0 + mm < M) st_word(src + (int64_t)mm * kBM, 0ull);     // empty again
                }
              }
            }
            if (n < N && ok_all) {
#pragma unroll
              for (int cb = 0; cb < (BN + 31) / 32; ++cb)
#pragma unroll
                for (int i = 0; i < kCols; ++i) {
                  const int64_t mm = q0 + cb * 32 + i;
                  if (mm < M) store_out(mm, __fmul_rn(sum[cb][i], alpha));
                }
            }
          }
        }
      }
      acc_phase ^= 1;
      acc_buf ^= 1;
      first_item = false;
    }
    if (tma_store && et == 0) bulk_wait_group<0>();   // stores done before the CTA's smem goes away
  } else {
    // ------------------------------------------------------------ scale copies
    // warp 6 copies P's scale chunks of each stage into TMEM, warp 7 + rb the
    // chunks of Q's 128-row block rb; each then commits to the stage's
    // scales-ready barrier (kCopyWarps arrivals).  A TMEM scale region is
    // rewritten only once the MMAs that read it last have completed.
    const bool copy_p = warp == 6;
    const int rbq = warp - 7;                   // Q block of this warp
    if (lane == 0 && leader) {                  // CTA pairs: the even CTA copies for both
      const uint64_t desc0 =
          smem_desc(sbase + (copy_p ? C::kOffSfa : (C::kQx ? C::kOffActSf : C::kOffSfb)), 16, 128, 0);
      const uint32_t sf_t0 = tmem_base + C::kSfBase;
      const int kc = p.kc;
      int stage = 0, region = 0;
      int64_t step = 0;                         // pipeline steps issued so far
      uint32_t phase = 0;
      bool ok = true;
      WorkIter w = work_begin(p, SWAP, PAIR);
      int tp, tq, kb0, ke0;
      while (ok && work_next(p, w, tp, tq, kb0, ke0)) {
        for (int k = kb0; k < ke0; ++k) {
          if (C::kQx && step >= C::kActSteps) { ok = false; break; }
          // in-kernel activation: this step's scales are written by the epilogue warps
          if (C::kQx && !copy_p && !mbar_wait(bar_act + 8 * (int)step, 0, abort_flag, p.err, p.timeout_ns)) {
            ok = false;
            break;
          }
          if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, p.err, p.timeout_ns)) { ok = false; break; }
          if (C::kSfRegions < C::kStages && step >= C::kSfRegions) {
            // the MMAs of step - kSfRegions read this region: wait for their
            // commit on that step's empty barrier (the full barrier above
            // already covers steps at least kStages back)
            const int64_t s2 = step - C::kSfRegions;
            if (!mbar_wait(bar_empty + 8 * (int)(s2 % C::kStages), (uint32_t)((s2 / C::kStages) & 1), abort_flag, p.err,
                           p.timeout_ns)) { ok = false; break; }
            tc_fence_after();
          }
          const uint32_t sfa_t = sf_t0 + region * C::kSfStageCols;
          const int nch = min(C::kChunks, kc - C::kChunks * k);
          if (copy_p) {
            const uint64_t d = desc0 + (uint64_t)((stage * C::kSfaBytes) >> 4);
            if constexpr (PAIR) {
              for (int c = 0; c < nch; ++c)
                tc_cp_32x128b_warpx4_pair(sfa_t + c * 4, d + (uint64_t)(c * (kSfChunk >> 4)));
            } else if (nch == C::kChunks) {
#pragma unroll
              for (int c = 0; c < C::kChunks; ++c)
                tc_cp_32x128b_warpx4(sfa_t + c * 4, d + (uint64_t)(c * (kSfChunk >> 4)));
            } else {
              for (int c = 0; c < nch; ++c) tc_cp_32x128b_warpx4(sfa_t + c * 4, d + (uint64_t)(c * (kSfChunk >> 4)));
            }
          } else {
            const uint64_t d = desc0 + (uint64_t)((C::kQx ? step * C::kActSfBytes : stage * C::kSfbBytes) >> 4);
            const uint32_t sfb_t = sfa_t + C::kSfaCols;
            for (int c = 0; c < nch; ++c) {
              if constexpr (PAIR)
                tc_cp_32x128b_warpx4_pair(sfb_t + c * 4 * C::kSfbBlocks + rbq * 4,
                                          d + (uint64_t)((rbq * C::kChunks + c) * (kSfChunk >> 4)));
              else
                tc_cp_32x128b_warpx4(sfb_t + c * 4 * C::kSfbBlocks + rbq * 4,
                                     d + (uint64_t)((rbq * C::kChunks + c) * (kSfChunk >> 4)));
            }
          }
          if constexpr (PAIR) tc_commit_pair(bar_sf + 8 * stage);
          else tc_commit(bar_sf + 8 * stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1; }
          if (++region == C::kSfRegions) region = 0;
          ++step;
        }
      }
      // every copy issued by this thread has landed before TMEM is freed
      const uint32_t db = bar_cp_drain + 8 * (warp - 6);
      if constexpr (PAIR) tc_commit_pair(db);
      else tc_commit(db);
      volatile int never = 0;
      (void)mbar_wait(db, 0, &never, p.err, p.drain_ns);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // no CTA of a cluster leaves while another may still write into, or read
  // from, its shared memory or TMEM (CTA pairs: the even CTA's tensor-core
  // work on both has drained)
  if constexpr (PAIR) cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemAlloc);
    else tmem_dealloc(tmem_base, C::kTmemAlloc);
  }
}

// ---------------------------------------------------------------- host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
    else
      (void)cudaGetLastError();
  });
  return fn;
}

// Codes of a [rows, K/2]-byte operand in boxes of row_bytes x box_rows, with
// the matching swizzle (128-byte rows: 128B, 64-byte rows: 64B).
bool make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int box_rows, int row_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Block scales in the tensor-core order viewed as [chunks, 128] 32-bit words
// (one 512-byte chunk per row), boxes of `chunks` consecutive chunks.
bool make_sf_map(CUtensorMap* m, const void* base, int64_t rows, int64_t kc, int chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {128, (cuuint64_t)(ceil_div(rows, 128) * kc)};
  const cuuint64_t strides[1] = {512};
  const cuuint32_t box[2] = {128, (cuuint32_t)chunks};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output [M, N] (bf16 or f32), boxes of 128 rows x 128 bytes, 128B swizzle.
bool make_out_map(CUtensorMap* m, void* base, int64_t M, int64_t N, bool f32) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int64_t esz = f32 ? 4 : 2;
  const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)(N * esz)};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)kBM};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Memory the caller declared read-only for the duration of library calls
// (nvfp4_declare_static): a GEMM whose weight codes and scales lie inside it
// loads its first weight stages before waiting on the preceding kernel.
std::mutex g_static_mu;
std::vector<std::pair<uintptr_t, uintptr_t>> g_static_ranges;   // [begin, end)

bool is_static(const void* p, size_t bytes) {
  const uintptr_t b = reinterpret_cast<uintptr_t>(p), e = b + bytes;
  std::lock_guard<std::mutex> lock(g_static_mu);
  for (const auto& r : g_static_ranges)
    if (b >= r.first && e <= r.second) return true;
  return false;
}

// Swapped (decode) tiles are split over the CTAs along K; partial tiles are
// exchanged through a K-split workspace of one stream: either one the caller
// registered for that stream (nvfp4_set_workspace: caller-owned, never freed
// here) or, failing that, one the library allocates on the first swapped
// call on that stream (all words empty) and frees in
// nvfp4_release_workspaces().  One per stream, because calls on unordered
// streams may run at the same time and must not share partial words.
struct Workspace {
  uint64_t* ws = nullptr;
  size_t bytes = 0;
  bool owned = false;   // allocated (and freed) by the library
};

std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws_table;

// CTAs of a swapped GEMM's grid, at most (Cfg::kGridPerSm per SM; the
// NVFP4 bound, which also covers the MXFP4 grid).
int64_t swap_grid_cap(const DeviceInfo* d, int bn) { return (int64_t)d->sm_count * (bn <= 16 ? 2 : 1); }

// Bytes of K-split workspace a swapped GEMM with activation side bn needs:
// two slots of bn x 128 words per CTA.
size_t workspace_need(const DeviceInfo* d, int bn) {
  return (size_t)2 * (size_t)swap_grid_cap(d, bn) * (size_t)bn * kBM * sizeof(uint64_t);
}

cudaError_t get_workspace(const DeviceInfo* d, cudaStream_t st, int bn, Workspace* out) {
  std::lock_guard<std::mutex> lock(g_ws_mu);
  auto it = g_ws_table.find({d->device, st});
  if (it != g_ws_table.end()) {
    if (it->second.bytes < workspace_need(d, bn)) return cudaErrorInvalidValue;   // a registered one too small
    *out = it->second;
    return cudaSuccess;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) return cudaErrorNotPermitted;
  Workspace w;
  w.bytes = workspace_need(d, 128);
  w.owned = true;
  cudaError_t e = cudaMalloc(&w.ws, w.bytes);
  if (e != cudaSuccess) return e;
  e = cudaMemset(w.ws, 0, w.bytes);
  if (e != cudaSuccess) {
    cudaFree(w.ws);
    return e;
  }
  g_ws_table[{d->device, st}] = w;
  *out = w;
  return cudaSuccess;
}

template <int BN, bool SWAP, bool OUT_F32, int QX = 0, bool MX = false, bool PAIR = false>
cudaError_t set_smem_attr(const DeviceInfo* d) {
  using Cf = Cfg<BN, SWAP, QX, MX, PAIR>;
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  std::call_once(once[d->device], [&] {
    auto kern = nvfp4_gemm_kernel<BN, SWAP, OUT_F32, QX, MX, PAIR>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmemBytes);
    // all of the SM's unified memory as shared memory: two co-resident CTAs
    // of 114 KB fit only with the full carveout, and a cooperative launch is
    // admitted against this preference
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    attr_err[d->device] = e;
  });
  return attr_err[d->device];
}

// CTAs of this kernel that can be resident on one SM (occupancy API, with the
// attributes set above), once per device; 0 if the query fails.
template <int BN, bool SWAP, bool OUT_F32, int QX = 0, bool MX = false, bool PAIR = false>
int resident_per_sm(const DeviceInfo* d) {
  using Cf = Cfg<BN, SWAP, QX, MX, PAIR>;
  static std::once_flag once[64];
  static int occ[64];
  std::call_once(once[d->device], [&] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4_gemm_kernel<BN, SWAP, OUT_F32, QX, MX, PAIR>,
                                                      Cf::kThreads, Cf::kSmemBytes) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    occ[d->device] = n;
  });
  return occ[d->device];
}

// grid: number of CTAs (0 = the persistent grid); cluster: CTAs per cluster
template <int BN, bool SWAP, bool OUT_F32, int QX = 0, bool MX = false, bool PAIR = false>
cudaError_t launch(const GemmParams& p, const DeviceInfo* d, cudaStream_t st, int grid = 0, int cluster = 1) {
  using Cf = Cfg<BN, SWAP, QX, MX, PAIR>;
  auto kern = nvfp4_gemm_kernel<BN, SWAP, OUT_F32, QX, MX, PAIR>;
  const cudaError_t ea = set_smem_attr<BN, SWAP, OUT_F32, QX, MX, PAIR>(d);
  if (ea != cudaSuccess) return ea;
  if (grid == 0) {
    if (SWAP) {
      const int64_t units = (int64_t)p.tiles_p * p.kt;
      int per_sm = Cf::kGridPerSm;
      if (decode_cooperative()) {
        // a cooperative grid must be resident at once: at most what the
        // occupancy API admits per SM
        const int occ = resident_per_sm<BN, SWAP, OUT_F32, QX, MX, PAIR>(d);
        if (occ < per_sm) per_sm = occ < 1 ? 1 : occ;
      }
      const int64_t cap = (int64_t)d->sm_count * per_sm;
      grid = (int)(units < cap ? units : cap);
    } else {
      const int tiles = p.tiles_p * p.tiles_q;
      grid = tiles < d->sm_count ? tiles : d->sm_count;
    }
  }
  // programmatic dependent launch: the kernel may start while the previous
  // kernel in the stream finishes; it waits (griddepcontrol.wait) before
  // touching anything that kernel produced
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Cf::kThreads);
  cfg.dynamicSmemBytes = Cf::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // split-K tiles: a tile's first CTA waits for partials from later CTAs,
  // so the grid (at most one CTA per SM) must be resident at once; opted in,
  // the driver guarantees that or refuses the launch
  if (SWAP && decode_cooperative()) {
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.numAttrs = 2;
  }
  if (PAIR) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  return cudaLaunchKernelEx(&cfg, kern, p);
}

float alpha_of(float ga, float gw) { return (float)(1.0 / ((double)ga * (double)gw)); }

template <bool MX>
cudaError_t launch_shape(const GemmParams& p, const DeviceInfo* d, cudaStream_t st, bool swap, int bn, bool f32) {
  if (!swap) {
    // CTA pairs: 256 x 256 tiles, a persistent grid of whole pairs
    const int64_t tiles = (int64_t)p.tiles_p * p.tiles_q;
    const int pairs = (int)(tiles < d->sm_count / 2 ? tiles : d->sm_count / 2);
    return f32 ? launch<256, false, true, 0, MX, true>(p, d, st, 2 * pairs, 2)
               : launch<256, false, false, 0, MX, true>(p, d, st, 2 * pairs, 2);
  }
  if (bn == 16) return f32 ? launch<16, true, true, 0, MX>(p, d, st) : launch<16, true, false, 0, MX>(p, d, st);
  if (bn == 32) return f32 ? launch<32, true, true, 0, MX>(p, d, st) : launch<32, true, false, 0, MX>(p, d, st);
  if (bn == 64) return f32 ? launch<64, true, true, 0, MX>(p, d, st) : launch<64, true, false, 0, MX>(p, d, st);
  return f32 ? launch<128, true, true, 0, MX>(p, d, st) : launch<128, true, false, 0, MX>(p, d, st);
}

// mx: MXFP4 operands (E8M0 scales of 32-element blocks, in the same chunk
// order with 4 scales = 128 K-elements per chunk); the caller passes unit
// global scales, so alpha = 1.
nvfp4_status run_gemm(const uint8_t* a_codes, const uint8_t* a_scales, float ga, const uint8_t* w_codes,
                      const uint8_t* w_scales, const int64_t* seg_offsets, const float* seg_gs, int n_seg,
                      int64_t M, int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype, cudaStream_t st,
                      bool mx = false, int test_stall = 0) {
  if (!a_codes || !a_scales || !w_codes || !w_scales || !out) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_INVALID_ARG;
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31)) return NVFP4_ERR_UNSUPPORTED;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
  if (!finite_positive(ga)) return NVFP4_ERR_INVALID_ARG;
  if (n_seg < 1 || n_seg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < n_seg; ++i)
    if (!finite_positive(seg_gs[i]) || seg_offsets[i + 1] <= seg_offsets[i]) return NVFP4_ERR_INVALID_ARG;
  if (seg_offsets[0] != 0 || seg_offsets[n_seg] != N) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(out))
    return NVFP4_ERR_ALIGNMENT;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  if (d->major != 10) return NVFP4_ERR_UNSUPPORTED;

  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const bool f32 = out_dtype == NVFP4_OUT_F32;
  p.err = d->err_word;
  p.timeout_ns = wait_timeout_ns();
  p.drain_ns = drain_timeout_ns();
  p.M = M;
  p.N = N;
  p.n_seg = n_seg;
  p.test_stall = test_stall;
  for (int i = 0; i < n_seg; ++i) {
    p.seg_end[i] = (int)seg_offsets[i + 1];
    p.seg_alpha[i] = alpha_of(ga, seg_gs[i]);
  }
  p.w_static = is_static(w_codes, (size_t)N * (size_t)(K / 2)) &&
                       is_static(w_scales, nvfp4_scale_bytes(N, mx ? K / 2 : K, NVFP4_SF_TCGEN05))
                   ? 1 : 0;
  p.kc = (int)ceil_div(K, mx ? 128 : 64);
  p.kmma = (int)ceil_div(K, 64);
  p.out = out;
  const bool swap = M <= 128;
  int bn = 256;
  if (swap) bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  if (swap) {
    Workspace w;
    const cudaError_t e = get_workspace(d, st, bn, &w);
    if (e == cudaErrorNotPermitted) return NVFP4_ERR_UNSUPPORTED;
    if (e == cudaErrorInvalidValue) return NVFP4_ERR_INVALID_ARG;
    if (e != cudaSuccess) return cuda_status(e);
    p.ws = w.ws;
    p.ws_words = w.bytes / sizeof(uint64_t);
  }
  p.rows_p = (int)(swap ? N : M);
  p.rows_q = (int)(swap ? M : N);
  const uint8_t* codes_p = swap ? w_codes : a_codes;
  const uint8_t* codes_q = swap ? a_codes : w_codes;
  p.sf_p = swap ? w_scales : a_scales;
  p.sf_q = swap ? a_scales : w_scales;
  const int kkb = swap ? Cfg<16, true>::kKB : Cfg<256, false>::kKB;
  // normal tiles run as CTA pairs: each CTA loads 128 rows of the 256-row
  // weight tile, and the scale chunks through tensor maps
  if (!make_code_map(&p.tmap_p, codes_p, p.rows_p, K, kBM, 32 * kkb) ||
      !make_code_map(&p.tmap_q, codes_q, p.rows_q, K, swap ? bn : kBM, 32 * kkb))
    return NVFP4_ERR_CUDA;
  if (!swap) {
    const int chunks = mx ? Cfg<256, false, 0, true>::kChunks : Cfg<256, false>::kChunks;
    if (!make_sf_map(&p.tmap_sfa, p.sf_p, p.rows_p, p.kc, chunks) ||
        !make_sf_map(&p.tmap_sfb, p.sf_q, p.rows_q, p.kc, chunks))
      return NVFP4_ERR_CUDA;
  }
  // TMA stores need 16-byte aligned output rows
  p.tma_store = (!swap && (N * (f32 ? 4 : 2)) % 16 == 0) ? 1 : 0;
  if (p.tma_store && !make_out_map(&p.tmap_out, out, M, N, f32)) return NVFP4_ERR_CUDA;
  p.rb_q = (int)ceil_div(p.rows_q, 128);
  p.sf_p_bytes = (uint64_t)ceil_div(p.rows_p, 128) * p.kc * kSfChunk;
  p.sf_q_bytes = (uint64_t)p.rb_q * p.kc * kSfChunk;
  p.out_elems = (uint64_t)M * (uint64_t)N;
  p.kt = (int)ceil_div(K, 64 * kkb);
  p.tiles_p = (int)ceil_div(p.rows_p, swap ? kBM : 2 * kBM);
  p.tiles_q = (int)ceil_div(p.rows_q, bn);
  p.group_p = swap ? kGroupP : kGroupP / 2;
  return cuda_status(mx ? launch_shape<true>(p, d, st, swap, bn, f32) : launch_shape<false>(p, d, st, swap, bn, f32));
}

// ---------------------------------------------------------------------------
// Allocation-free decode GEMM (nvfp4_gemm_noalloc).  Same kernel and same
// work split as the swapped (M <= 128) path of nvfp4_gemm, but its K-split
// scratch is a fixed array in this module's static device memory instead of
// the per-stream workspace nvfp4_gemm allocates on first use.  It serves
// callers that must not allocate device memory after start-up: a serving
// engine that measures its peak memory once and hands the remainder to its
// KV cache (a later allocation can fail or eat into that cache), and code
// that cannot afford the implicit device synchronisation cudaMalloc may
// perform.
//
// Limits (the scratch is sized for them; larger inputs are rejected with
// NVFP4_ERR_UNSUPPORTED): M <= 32, at most 160 SMs.  Scratch: tagged partial
// tiles, 2 slots x 160 CTAs x (32 x 128) 64-bit words = 10 MiB.  Every word
// must be empty (zero) when a launch starts: the array is zero-initialised
// when the module loads, each launch leaves every word it used empty, and
// after a launch that timed out nvfp4_last_device_error() clears it.
constexpr int kNoAllocMaxM = 32;
constexpr int kNoAllocMaxCtas = 160;
constexpr size_t kNoAllocScratchBytes = (size_t)2 * kNoAllocMaxCtas * kNoAllocMaxM * kBM * sizeof(uint64_t);

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address on each device, resolved on the first call on
// that device with it current.  Only a successful lookup is kept, so a lookup
// that failed (for example a lazy module load under memory pressure) is tried
// again on the next call.  The address is published with release order and
// read with acquire order (clear_gemm_scratch reads it from any thread).
struct NoAllocScratch {
  std::mutex mu;
  std::atomic<uint8_t*> ptr{nullptr};
};
NoAllocScratch g_noalloc[64];

uint8_t* noalloc_scratch_ptr(int device) {
  NoAllocScratch& sc = g_noalloc[device];
  uint8_t* p = sc.ptr.load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(sc.mu);
  p = sc.ptr.load(std::memory_order_relaxed);
  if (p) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) {
    (void)cudaGetLastError();
    return nullptr;
  }
  p = static_cast<uint8_t*>(addr);
  sc.ptr.store(p, std::memory_order_release);
  return p;
}

// Quantize X then multiply.  Given activation buffers, the quantize kernel
// writes (a_codes, a_scales) and the GEMM reads them.  Without them,
// decode-sized M runs as one kernel whose epilogue warps quantize X into
// shared memory before the first MMA.  (That one-kernel form measured slower
// than the two kernels on the decode shape: every CTA quantizes the part of
// X its K range needs, so X is quantized many times over, in four warps that
// cannot hide latency, whereas the quantize kernel spreads X over the whole
// GPU once.)
constexpr int kLinearMaxM = 32;

bool linear_fused_fits(const DeviceInfo* d, int64_t M, int64_t N, int64_t K) {
  if (M > kLinearMaxM) return false;
  const int bn = M <= 16 ? 16 : 32;
  const int64_t units = ceil_div(N, kBM) * ceil_div(K, 64 * Cfg<16, true>::kKB);
  // a cooperative grid may be as small as one CTA per SM (see launch())
  const int64_t cap = decode_cooperative() ? (int64_t)d->sm_count : swap_grid_cap(d, bn);
  const int64_t grid = units < cap ? units : cap;
  const int steps = bn == 16 ? Cfg<16, true, 1>::kActSteps : Cfg<32, true, 1>::kActSteps;
  return ceil_div(units, grid) <= steps;   // steps per CTA, at most
}

template <int BN, int QX>
cudaError_t launch_linear(const GemmParams& p, const DeviceInfo* d, cudaStream_t st, bool f32) {
  return f32 ? launch<BN, true, true, QX>(p, d, st) : launch<BN, true, false, QX>(p, d, st);
}

nvfp4_status run_linear(const void* x, nvfp4_in_dtype x_dtype, int64_t M, int64_t K, float ga, const uint8_t* w_codes,
                        const uint8_t* w_scales, float gw, int64_t N, void* out, nvfp4_out_dtype out_dtype,
                        uint8_t* a_codes, uint8_t* a_scales, cudaStream_t st) {
  if (!x || !w_codes || !w_scales || !out) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_INVALID_ARG;
  if (x_dtype != NVFP4_IN_BF16 && x_dtype != NVFP4_IN_F32) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
  if (!finite_positive(ga) || !finite_positive(gw)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(out)) return NVFP4_ERR_ALIGNMENT;
  if (M > (1ll << 31) - 256 || N > (1ll << 31) - 256 || K > (1ll << 31)) return NVFP4_ERR_UNSUPPORTED;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  if (d->major != 10) return NVFP4_ERR_UNSUPPORTED;
  if ((a_codes && a_scales) || !linear_fused_fits(d, M, N, K)) {
    if (!a_codes || !a_scales) return NVFP4_ERR_INVALID_ARG;
    const nvfp4_status s1 = nvfp4_quantize(x, x_dtype, M, K, ga, a_codes, a_scales, NVFP4_SF_TCGEN05, nullptr, st);
    if (s1 != NVFP4_OK) return s1;
    return nvfp4_gemm(a_codes, a_scales, ga, w_codes, w_scales, gw, M, N, K, out, out_dtype, st);
  }
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int bn = M <= 16 ? 16 : 32;
  Workspace w;
  const cudaError_t e0 = get_workspace(d, st, bn, &w);
  if (e0 == cudaErrorNotPermitted) return NVFP4_ERR_UNSUPPORTED;
  if (e0 == cudaErrorInvalidValue) return NVFP4_ERR_INVALID_ARG;
  if (e0 != cudaSuccess) return cuda_status(e0);
  p.ws = w.ws;
  p.ws_words = w.bytes / sizeof(uint64_t);
  constexpr int kkb = Cfg<16, true>::kKB;
  p.rows_p = (int)N;
  p.rows_q = (int)M;
  p.sf_p = w_scales;
  p.sf_q = nullptr;
  if (!make_code_map(&p.tmap_p, w_codes, p.rows_p, K, kBM, 32 * kkb)) return NVFP4_ERR_CUDA;
  p.tmap_q = p.tmap_p;                      // not read (X is quantized in the kernel)
  p.w_static = is_static(w_codes, (size_t)N * (size_t)(K / 2)) &&
                       is_static(w_scales, nvfp4_scale_bytes(N, K, NVFP4_SF_TCGEN05))
                   ? 1 : 0;
  p.out = out;
  p.tma_store = 0;
  p.err = d->err_word;
  p.timeout_ns = wait_timeout_ns();
  p.drain_ns = drain_timeout_ns();
  p.M = M;
  p.N = N;
  p.rb_q = 1;
  p.kc = (int)ceil_div(K, 64);
  p.kmma = (int)ceil_div(K, 64);
  p.kt = (int)ceil_div(K, 64 * kkb);
  p.tiles_p = (int)ceil_div(p.rows_p, kBM);
  p.tiles_q = 1;
  p.n_seg = 1;
  p.seg_end[0] = (int)N;
  p.seg_alpha[0] = alpha_of(ga, gw);
  p.x = x;
  p.x_gs = ga;
  p.K = K;
  p.sf_p_bytes = (uint64_t)ceil_div(N, 128) * p.kc * kSfChunk;
  p.out_elems = (uint64_t)M * (uint64_t)N;
  p.x_bytes = (uint64_t)M * (uint64_t)K * (x_dtype == NVFP4_IN_F32 ? 4 : 2);
  const bool f32 = out_dtype == NVFP4_OUT_F32;
  const bool xf32 = x_dtype == NVFP4_IN_F32;
  cudaError_t e;
  if (bn == 16) e = xf32 ? launch_linear<16, 2>(p, d, st, f32) : launch_linear<16, 1>(p, d, st, f32);
  else e = xf32 ? launch_linear<32, 2>(p, d, st, f32) : launch_linear<32, 1>(p, d, st, f32);
  return cuda_status(e);
}

}  // namespace

// After a launch whose bounded wait ran out, partial words may be left full;
// empty every K-split scratch of the current device (library workspaces and
// the allocation-free scratch).  Synchronous.
cudaError_t clear_gemm_scratch(int device) {
  cudaError_t first = cudaSuccess;
  {
    std::lock_guard<std::mutex> lock(g_ws_mu);
    for (auto& kv : g_ws_table)
      if (kv.first.first == device) {
        const cudaError_t e = cudaMemset(kv.second.ws, 0, kv.second.bytes);
        if (first == cudaSuccess) first = e;
      }
  }
  uint8_t* na = device >= 0 && device < 64 ? g_noalloc[device].ptr.load(std::memory_order_acquire) : nullptr;
  if (na) {
    const cudaError_t e = cudaMemset(na, 0, kNoAllocScratchBytes);
    if (first == cudaSuccess) first = e;
  }
  const cudaError_t e = cudaDeviceSynchronize();
  return first == cudaSuccess ? e : first;
}

namespace {

nvfp4_status run_gemm_noalloc(const uint8_t* a_codes, const uint8_t* a_scales, float ga, const uint8_t* w_codes,
                              const uint8_t* w_scales, float gw, int64_t M, int64_t N, int64_t K, void* out,
                              nvfp4_out_dtype out_dtype, cudaStream_t st, int test_stall = 0) {
  if (!a_codes || !a_scales || !w_codes || !w_scales || !out) return NVFP4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
  if (!finite_positive(ga) || !finite_positive(gw)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(out))
    return NVFP4_ERR_ALIGNMENT;
  if (M > kNoAllocMaxM || N > (1ll << 31) - 256 || K > (1ll << 31)) return NVFP4_ERR_UNSUPPORTED;
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  if (d->major != 10 || d->sm_count > kNoAllocMaxCtas || d->device >= 64) return NVFP4_ERR_UNSUPPORTED;
  // with this device current (device_info() reads the current device): the
  // scratch array's address on it, looked up once and then cached
  uint8_t* scratch = noalloc_scratch_ptr(d->device);
  if (!scratch) return NVFP4_ERR_CUDA;

  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int bn = M <= 16 ? 16 : 32;
  // the grid's partial slots fit the scratch: 2 x (2 x SMs) x 16 x 128 words
  // for bn = 16, 2 x SMs x 32 x 128 for bn = 32; both fit for <= 160 SMs
  if (workspace_need(d, bn) > kNoAllocScratchBytes) return NVFP4_ERR_UNSUPPORTED;
  p.ws = reinterpret_cast<uint64_t*>(scratch);
  p.ws_words = kNoAllocScratchBytes / sizeof(uint64_t);
  p.rows_p = (int)N;
  p.rows_q = (int)M;
  p.sf_p = w_scales;
  p.sf_q = a_scales;
  constexpr int kkb = Cfg<16, true>::kKB;
  if (!make_code_map(&p.tmap_p, w_codes, p.rows_p, K, kBM, 32 * kkb) ||
      !make_code_map(&p.tmap_q, a_codes, p.rows_q, K, bn, 32 * kkb))
    return NVFP4_ERR_CUDA;
  p.out = out;
  p.tma_store = 0;
  p.err = d->err_word;
  p.timeout_ns = wait_timeout_ns();
  p.drain_ns = drain_timeout_ns();
  p.M = M;
  p.N = N;
  p.rb_q = (int)ceil_div(p.rows_q, 128);
  p.kc = (int)ceil_div(K, 64);
  p.kmma = (int)ceil_div(K, 64);
  p.kt = (int)ceil_div(K, 64 * kkb);
  p.tiles_p = (int)ceil_div(p.rows_p, kBM);
  p.tiles_q = 1;
  p.n_seg = 1;
  p.test_stall = test_stall;
  p.seg_end[0] = (int)N;
  p.seg_alpha[0] = alpha_of(ga, gw);
  p.sf_p_bytes = (uint64_t)ceil_div(N, 128) * p.kc * kSfChunk;
  p.sf_q_bytes = (uint64_t)p.rb_q * p.kc * kSfChunk;
  p.out_elems = (uint64_t)M * (uint64_t)N;
  cudaError_t e;
  const bool f32 = out_dtype == NVFP4_OUT_F32;
  if (bn == 16) e = f32 ? launch<16, true, true>(p, d, st) : launch<16, true, false>(p, d, st);
  else e = f32 ? launch<32, true, true>(p, d, st) : launch<32, true, false>(p, d, st);
  return cuda_status(e);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, float a_global_scale,
                        const uint8_t* w_codes, const uint8_t* w_scales, float w_global_scale, int64_t M, int64_t N,
                        int64_t K, void* out, nvfp4_out_dtype out_dtype, nvfp4_stream_t stream) {
  const int64_t offs[2] = {0, N};
  const float gs[1] = {w_global_scale};
  return run_gemm(a_codes, a_scales, a_global_scale, w_codes, w_scales, offs, gs, 1, M, N, K, out, out_dtype,
                  (cudaStream_t)stream);
}

size_t nvfp4_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 32 || K % 32 != 0) return 0;
  if (M > 128) return 0;                              // normal tiles do not split K
  const DeviceInfo* d = device_info();
  if (!d) return 0;
  const int bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  return workspace_need(d, bn);
}

nvfp4_status nvfp4_set_workspace(nvfp4_stream_t stream, void* workspace, size_t bytes) {
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  const cudaStream_t st = (cudaStream_t)stream;
  std::lock_guard<std::mutex> lock(g_ws_mu);
  auto it = g_ws_table.find({d->device, st});
  if (it != g_ws_table.end() && it->second.owned) {
    // a workspace the library allocated earlier for this stream: freed once
    // the device is idle
    if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
    cudaFree(it->second.ws);
    g_ws_table.erase(it);
  } else if (it != g_ws_table.end()) {
    g_ws_table.erase(it);
  }
  if (!workspace) return bytes == 0 ? NVFP4_OK : NVFP4_ERR_INVALID_ARG;   // unregistered
  if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
  if (bytes < workspace_need(d, 16)) return NVFP4_ERR_INVALID_ARG;
  Workspace w;
  w.ws = static_cast<uint64_t*>(workspace);
  w.bytes = bytes;
  w.owned = false;
  g_ws_table[{d->device, st}] = w;
  return NVFP4_OK;
}

nvfp4_status nvfp4_release_workspaces(void) {
  const DeviceInfo* d = device_info();
  if (!d) return NVFP4_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return cuda_status(cudaGetLastError());
  std::lock_guard<std::mutex> lock(g_ws_mu);
  for (auto it = g_ws_table.begin(); it != g_ws_table.end();) {
    if (it->first.first == d->device && it->second.owned) {
      cudaFree(it->second.ws);
      it = g_ws_table.erase(it);
    } else {
      ++it;
    }
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_declare_static(const void* base, size_t bytes) {
  if (!base || bytes == 0) return NVFP4_ERR_INVALID_ARG;
  const uintptr_t b = reinterpret_cast<uintptr_t>(base);
  std::lock_guard<std::mutex> lock(g_static_mu);
  g_static_ranges.emplace_back(b, b + bytes);
  return NVFP4_OK;
}

void nvfp4_forget_static(void) {
  std::lock_guard<std::mutex> lock(g_static_mu);
  g_static_ranges.clear();
}

nvfp4_status nvfp4_linear(const void* x, nvfp4_in_dtype x_dtype, int64_t M, int64_t K, float a_global_scale,
                          const uint8_t* w_codes, const uint8_t* w_scales, float w_global_scale, int64_t N, void* out,
                          nvfp4_out_dtype out_dtype, uint8_t* a_codes, uint8_t* a_scales, nvfp4_stream_t stream) {
  return run_linear(x, x_dtype, M, K, a_global_scale, w_codes, w_scales, w_global_scale, N, out, out_dtype, a_codes,
                    a_scales, (cudaStream_t)stream);
}

nvfp4_status nvfp4_fused_proj(const uint8_t* a_codes, const uint8_t* a_scales, float a_global_scale,
                              const uint8_t* w_codes, const uint8_t* w_scales, const int64_t* seg_offsets,
                              const float* seg_global_scales, int n_seg, int64_t M, int64_t K, void* out,
                              nvfp4_out_dtype out_dtype, nvfp4_stream_t stream) {
  if (!seg_offsets || !seg_global_scales || n_seg < 1 || n_seg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  return run_gemm(a_codes, a_scales, a_global_scale, w_codes, w_scales, seg_offsets, seg_global_scales, n_seg, M,
                  seg_offsets[n_seg], K, out, out_dtype, (cudaStream_t)stream);
}

nvfp4_status nvfp4_mx_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                           const uint8_t* w_scales, int64_t M, int64_t N, int64_t K, void* out,
                           nvfp4_out_dtype out_dtype, nvfp4_stream_t stream) {
  const int64_t offs[2] = {0, N};
  const float unit[1] = {1.0f};
  return run_gemm(a_codes, a_scales, 1.0f, w_codes, w_scales, offs, unit, 1, M, N, K, out, out_dtype,
                  (cudaStream_t)stream, /*mx=*/true);
}

nvfp4_status nvfp4_gemm_noalloc(const uint8_t* a_codes, const uint8_t* a_scales, float a_global_scale,
                                const uint8_t* w_codes, const uint8_t* w_scales, float w_global_scale, int64_t M,
                                int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype, nvfp4_stream_t stream) {
  return run_gemm_noalloc(a_codes, a_scales, a_global_scale, w_codes, w_scales, w_global_scale, M, N, K, out,
                          out_dtype, (cudaStream_t)stream);
}

nvfp4_status nvfp4_test_gemm_stalled_reduction(const uint8_t* a_codes, const uint8_t* a_scales, float a_global_scale,
                                               const uint8_t* w_codes, const uint8_t* w_scales, float w_global_scale,
                                               int64_t M, int64_t N, int64_t K, void* out, nvfp4_out_dtype out_dtype,
                                               int noalloc, nvfp4_stream_t stream) {
  if (M > 128) return NVFP4_ERR_UNSUPPORTED;                 // only decode tiles split K
  if (noalloc)
    return run_gemm_noalloc(a_codes, a_scales, a_global_scale, w_codes, w_scales, w_global_scale, M, N, K, out,
                            out_dtype, (cudaStream_t)stream, /*test_stall=*/1);
  const int64_t offs[2] = {0, N};
  const float gs[1] = {w_global_scale};
  return run_gemm(a_codes, a_scales, a_global_scale, w_codes, w_scales, offs, gs, 1, M, N, K, out, out_dtype,
                  (cudaStream_t)stream, /*mx=*/false, /*test_stall=*/1);
}

}  // extern "C"
