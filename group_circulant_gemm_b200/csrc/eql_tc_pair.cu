// Pair-CTA tcgen05 forward of the p4 (T = 4) EQ-Linear layer from spectral
// input planes, FP16 in, FP32 accumulate, FP16 out, for sm_100a.
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" items 1-3
// and "Specialisation for p4"): the input arrives as its group DFT, four FP16
// planes X0, X2, Xr, Xi (each times 1/4) in the tiled layout below; per
// frequency the real products against the prepared weight planes (A0, A2, Br,
// Bi):
//   Y0 = X0 A0^T,  Y2 = X2 A2^T,
//   Y1r = Xr Br^T - Xi Bi^T,  Y1i = Xr Bi^T + Xi Br^T
// (six products of N = 128; -Xi Bi^T through the instruction's negate-A bit),
// then the inverse DFT plus bias (and activation) in the epilogue, written as
// Y [N][Cout*4] or as the next layer's planes.
//
// Why a CTA pair: with one CTA per tile, an M = 128 MMA reads both operands
// from its own SM's shared memory at about the rate that memory delivers, so
// every byte the TMA writes or another warp moves slows the tensor core.  With
// tcgen05.mma.cta_group::2 two SMs compute a 256-row tile: each holds its own
// 128 rows of the A operand (the input planes) and half of the B rows (the
// weights), so each SM reads half the weight bytes and its TMA fetches half of
// the weight tile from L2.  The inputs are already transformed, so nothing but
// the TMA and the tensor core touches the operand ring.  With products of
// N = 128 each weight plane is split between the two SMs and loaded once (two
// N = 256 products [Br | Bi], [-Bi | Br] would need Br on both SMs): the main
// loop is bound by L2 -> SM bytes, 24 KB per SM per K step.
//
// Tiled planes (the layout of eqlinear_group_dft's output): the planes are
// stored in HBM exactly as the MMA reads them from shared memory, so every
// load is whole 128-byte lines (a TMA fetches a box line by line; 32-byte rows
// cost as many requests as 128-byte ones).  Rows are padded to Np, a multiple
// of 128; element (plane p, row n, channel c) sits at byte
//   ((p * (C / 16) + c / 16) * Np + n) * 32 + ((h ^ ((n / 4) % 2)) * 16) + (c % 8) * 2,
// h = (c % 16) / 8: per 16-channel block, 32-byte rows with the 32-byte
// swizzle of the MMA's K-major operand layout.
//
// Design (cluster of 2 CTAs, one per SM, persistent over (256-row, 128
// out-channel) tiles; K step = 16 input channels, stage = 2 K steps):
//   warp 0    producer (both CTAs): per stage one 4-D TMA box of the tiled
//             planes (2 channel blocks x 128 own rows x 4 planes = 32 KB) and one
//             box of this CTA's half of the weights (16 KB), both completing on
//             the leader CTA's stage barrier (cta_group::2 loads).
//   warps 1, 3 TMEM allocation (warp 1, both CTAs); lane 0 of warps 1 and 3 of
//             the leader issue the six pair MMAs of each K step, three each, and
//             each commits its stage releases to both CTAs.  A tcgen05.mma costs
//             its issuing thread about 70 cycles, about what an N = 128 pair MMA
//             keeps the tensor core busy; two issuers and two K steps per stage
//             (one barrier wait and one commit) keep the issue ahead of it.
//   warps 4-11 epilogue (both CTAs, own 128 rows): read the tile's four FP32
//             accumulators from TMEM, inverse DFT + bias (+ activation; with
//             no activation, output as the next layer's planes is the
//             accumulators' frequencies plus the bias), pack to FP16; the
//             first 16 out-channels go to the staging buffer and the other 48
//             stay in registers, so TMEM is handed back to the MMA issuer before
//             any store drains; then four TMA stores of 32 rows x 16 channels.
// TMEM per CTA: Y0 [0,128) | Y2 [128,256) | Y1r [256,384) | Y1i [384,512).
// Every wait is bounded (about 2 s); on expiry the CTA sets its abort flag and
// the plan's status word, drains what it issued, and both CTAs meet at the
// final cluster barrier, so a stuck pipeline never hangs the GPU.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"
#include "eql_tc_fwd_parts.cuh"
#include "eql_tc_pair_common.cuh"

namespace eql {
namespace {

using namespace tc;
using namespace ftc;

constexpr int PR_BD = 128;                       // out-channels per tile
constexpr int PR_KC = 16;                        // input channels per K step
constexpr int PR_KSS = 2;                        // K steps per stage (32 channels)
constexpr int PR_ROWB = 32;                      // bytes per operand row (16 halves)
constexpr uint32_t PR_XBLK = BM * PR_ROWB;       // 4 KB: one plane, one K step, own 128 rows
constexpr uint32_t PR_XPLANE = PR_KSS * PR_XBLK;  // 8 KB: one plane of a stage
constexpr uint32_t PR_XBYTES = 4 * PR_XPLANE;    // 32 KB
constexpr int PR_WROWS = 256;                    // this CTA's weight rows per K step
constexpr uint32_t PR_WKS = PR_WROWS * PR_ROWB;  // 8 KB per K step
constexpr uint32_t PR_WBYTES = PR_KSS * PR_WKS;  // 16 KB per stage
constexpr int PR_WLINES = PR_WBYTES / 128;       // the weight stage as 128-byte lines
constexpr uint32_t PR_STAGE = PR_XBYTES + PR_WBYTES;  // 48 KB
constexpr int PR_ST = 4;                         // ring depth
// warps: 0 producer, 1 TMEM + MMA issuer, 2 idle, 3 MMA issuer, 4-11 epilogue
// (lane quarter = warp % 4); 168 registers a thread (three warps per SM
// sub-partition)
constexpr int PR_THREADS = 384;
constexpr int PR_EPI0 = 4;
constexpr uint32_t PR_OFF_STG = PR_ST * PR_STAGE;
constexpr uint32_t PR_OFF_BIAS = PR_OFF_STG + kEpiWarps * kStgBytes;
constexpr uint32_t PR_OFF_BAR = PR_OFF_BIAS + kEpiWarps * 128;
constexpr uint32_t PR_SMEM = PR_OFF_BAR + 512 + 1024;
static_assert(PR_STAGE % 1024 == 0, "stage slots stay 1024-byte aligned");
static_assert(PR_SMEM <= 232448, "shared memory budget");
// weight regions of a K step: this CTA's 64 rows (out-channels 64 * rank ..) of
// A0, A2, Br, Bi, each 64 x 32 B (a narrow tile: 32 rows each, out-channels
// 32 * rank ..)

struct PairBars {
  uint64_t full[PR_ST];   // leader: both CTAs' bytes of a stage landed
  uint64_t empty[PR_ST];  // each CTA: the stage's MMAs are done (multicast commit)
  uint64_t acc_full;      // each CTA: the tile's accumulators are final
  uint64_t acc_empty;     // leader: both CTAs' epilogues have read TMEM
  uint64_t drain[2];      // leader: every MMA an issuer issued is complete
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(PairBars) <= 512, "barrier block");

// Stores of the next layer's tiled planes: 32 rows (row0 a multiple of 32) x 16
// channels x 4 planes, one 4-D box; rows of the padding past N are written too
// (they belong to the buffer), tiles wholly past N are skipped.
struct TiledStore {
  const CUtensorMap* map;
  int64_t row0, N;
  __device__ __forceinline__ void operator()(uint32_t src, int d0) const {
    if (row0 < N) tma_store_4d(map, src, 0, (int)(row0 / 4), d0 / 16, 0);
  }
};
template <int IO>
using PairStoreOf = typename std::conditional<IO == kIoSpectralOut, TiledStore, RowStore<4>>::type;

// Two 8-channel slices (16 out-channels) of this lane's row into the warp's
// staging buffer, in the layout of one TMA store box: spatial Y (32 rows x
// 128 B, 128-byte swizzle) or spectral planes ([plane][32 rows][32 B], 32-byte
// swizzle).
template <int IO>
__device__ __forceinline__ void stage_two(uint8_t* stg, int lane, const uint4 (&a)[4],
                                          const uint4 (&b)[4]) {
  if constexpr (IO == kIoSpectralOut) {
    const int sw = (lane >> 2) & 1;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      *reinterpret_cast<uint4*>(stg + p * 1024 + lane * 32 + ((0 ^ sw) << 4)) = a[p];
      *reinterpret_cast<uint4*>(stg + p * 1024 + lane * 32 + ((1 ^ sw) << 4)) = b[p];
    }
  } else {
    uint8_t* row = stg + lane * 128;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      *reinterpret_cast<uint4*>(row + ((m ^ (lane & 7)) << 4)) = a[m];
      *reinterpret_cast<uint4*>(row + (((4 + m) ^ (lane & 7)) << 4)) = b[m];
    }
  }
}

// One 8-channel slice of this lane's row: the four accumulator planes
// (columns p * 128 + c0 .. +8) -> 64 bytes of output.  Both operands carry 1/4,
// so the accumulators hold Y/16; the inverse transform's terms are 4 acc (real
// frequencies) and 8 acc (complex), folded into FMAs (the products by powers of
// two are exact, so each result equals the separate multiply and add).
__device__ __forceinline__ void slice_load(uint32_t lane_addr, int c0, uint32_t (&v)[4][8]) {
#pragma unroll
  for (int p = 0; p < 4; ++p) tmem_ld_32x32b<8>(lane_addr + p * PR_BD + c0, v[p]);
}
template <int ACT>
__device__ __forceinline__ uint64_t f2_act(uint64_t v) {
  if constexpr (ACT == 0) {
    return v;
  } else {
    float lo, hi;
    f2_unpack(v, lo, hi);
    return f2_pack(act_fn<ACT>(lo), act_fn<ACT>(hi));
  }
}

template <int IO, int ACT>
__device__ __forceinline__ void slice_compute(const uint32_t (&v)[4][8], const __half* bs,
                                              uint4 (&o)[4]) {
  const uint4 bb = *reinterpret_cast<const uint4*>(bs);
  const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
  const uint64_t k4 = f2_pack(4.f, 4.f), km4 = f2_pack(-4.f, -4.f);
  const uint64_t k8 = f2_pack(8.f, 8.f), km8 = f2_pack(-8.f, -8.f);
  uint32_t w[4][4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    // channels 2m, 2m+1 as the two lanes
    const float2 bf = unpack_h2(bw[m]);
    const uint64_t a0 = f2_pack(__uint_as_float(v[0][2 * m]), __uint_as_float(v[0][2 * m + 1]));
    const uint64_t a2 = f2_pack(__uint_as_float(v[1][2 * m]), __uint_as_float(v[1][2 * m + 1]));
    const uint64_t ar = f2_pack(__uint_as_float(v[2][2 * m]), __uint_as_float(v[2][2 * m + 1]));
    const uint64_t ai = f2_pack(__uint_as_float(v[3][2 * m]), __uint_as_float(v[3][2 * m + 1]));
    const uint64_t sb = f2_fma(k4, a0, f2_pack(bf.x, bf.y));
    const uint64_t ev = f2_fma(k4, a2, sb), od = f2_fma(km4, a2, sb);
    if constexpr (IO == kIoSpectralOut && ACT == 0) {
      // No activation between this layer's inverse DFT and the next layer's
      // forward DFT: the two cancel, and the next layer's planes (times 1/4) are
      // the accumulators' frequencies themselves,
      //   (sum_s y_s)/4 = 4 a0 + b,  (y0 - y1 + y2 - y3)/4 = 4 a2,
      //   (y0 - y2)/4 = 4 ar,        (y3 - y1)/4 = 4 ai
      // (y_s as below; the products by 4 are exact): one rounding to FP16.
      float lo, hi;
      f2_unpack(sb, lo, hi); w[0][m] = pack_h2(lo, hi);
      f2_unpack(f2_mul(k4, a2), lo, hi); w[1][m] = pack_h2(lo, hi);
      f2_unpack(f2_mul(k4, ar), lo, hi); w[2][m] = pack_h2(lo, hi);
      f2_unpack(f2_mul(k4, ai), lo, hi); w[3][m] = pack_h2(lo, hi);
      continue;
    }
    uint64_t z0 = f2_act<ACT>(f2_fma(k8, ar, ev));
    uint64_t z1 = f2_act<ACT>(f2_fma(km8, ai, od));
    uint64_t z2 = f2_act<ACT>(f2_fma(km8, ar, ev));
    uint64_t z3 = f2_act<ACT>(f2_fma(k8, ai, od));
    if constexpr (IO == kIoSpectralOut) {
      // the next layer's planes (times 1/4): o[p] holds plane p of the 8 channels
      const uint64_t q = f2_pack(0.25f, 0.25f);
      const uint64_t a = f2_add(z0, z2), b = f2_add(z1, z3);
      const uint64_t p0 = f2_mul(f2_add(a, b), q), p1 = f2_mul(f2_sub(a, b), q);
      const uint64_t p2 = f2_mul(f2_sub(z0, z2), q), p3 = f2_mul(f2_sub(z3, z1), q);
      float lo, hi;
      f2_unpack(p0, lo, hi); w[0][m] = pack_h2(lo, hi);
      f2_unpack(p1, lo, hi); w[1][m] = pack_h2(lo, hi);
      f2_unpack(p2, lo, hi); w[2][m] = pack_h2(lo, hi);
      f2_unpack(p3, lo, hi); w[3][m] = pack_h2(lo, hi);
    } else {
      // channel 2m + e: four outputs y0..y3, contiguous in Y
      float y0[2], y1[2], y2[2], y3[2];
      f2_unpack(z0, y0[0], y0[1]);
      f2_unpack(z1, y1[0], y1[1]);
      f2_unpack(z2, y2[0], y2[1]);
      f2_unpack(z3, y3[0], y3[1]);
      w[m][0] = pack_h2(y0[0], y1[0]);
      w[m][1] = pack_h2(y2[0], y3[0]);
      w[m][2] = pack_h2(y0[1], y1[1]);
      w[m][3] = pack_h2(y2[1], y3[1]);
    }
  }
  if constexpr (IO == kIoSpectralOut) {
#pragma unroll
    for (int p = 0; p < 4; ++p) o[p] = make_uint4(w[p][0], w[p][1], w[p][2], w[p][3]);
  } else {
    // 16-byte piece m = channels 2m, 2m+1
#pragma unroll
    for (int m = 0; m < 4; ++m) o[m] = make_uint4(w[m][0], w[m][1], w[m][2], w[m][3]);
  }
}

// ---------------------------------------------------------------------------
// Work: a task is one (256-row block, 128 out-channel) tile of a layer.  One
// layer: the pair takes tiles pair, pair + npairs, ... (every role walks the
// same list).  Two chained layers (H = act(L1(X)) as tiled planes, Y = L2(H)):
// the tiles of both layers form one queue taken through a global counter; the
// leader's producer takes a task and hands it to every role of both CTAs
// through a small ring in each CTA's shared memory (the id is written to the
// peer with a cluster store, then the peer's ring barrier gets a remote
// arrive); a layer-2 tile waits (bounded) until its row block's layer-1 tiles
// are stored, counted per row block by the epilogue warps.
// ---------------------------------------------------------------------------
constexpr int kPQ = 4;  // task ring depth
// readers of a ring slot (arriving on the leader's empty barrier): leader's two
// issuers and 8 epilogue warps, the peer's producer and 8 epilogue warps
constexpr int kPRingReaders = 2 + kEpiWarps + 1 + kEpiWarps;

struct PairRing {
  uint64_t full[kPQ];   // each CTA: the slot's id is written
  uint64_t empty[kPQ];  // leader: every reader of both CTAs has the id
  int id[kPQ];
};
static_assert(sizeof(PairBars) + sizeof(PairRing) <= 512, "barrier block");

struct PairLayer {
  int n_dt;   // out-channel tiles
  int n_ks;   // stages of 32 input channels
  int Cout;
  int narrow;        // the last out-channel tile holds <= 64 channels: N = 64 products
  int narrow_line0;  // weight-tile line where that tile's stages start
  const __half* bias;
};
// The last out-channel tile of a layer whose remainder is at most 64 channels
// runs N = 64 products (each SM 32 weight rows per plane): half the weight bytes
// and tensor time of a zero-padded 128-channel tile.
__device__ __forceinline__ bool pair_narrow(const PairLayer& L, int dt) {
  return L.narrow && dt == L.n_dt - 1;
}
struct PairSched {
  int64_t N;
  int n_prow;        // 256-row blocks
  int total;         // tasks
  int lag;           // (chain) layer-1 row blocks queued ahead of layer 2
  int flag_target;   // (chain) counter value of a complete layer-1 row block
  int npairs;        // (chain) clusters in the grid
  PairLayer L[2];
};
struct PairTask {
  int layer, prow, dt;
};

// One layer: task u = (prow, dt) of layer 0, the full 128-channel tiles of every
// row block first and a narrow last tile's tasks after them, so a pair that takes
// a second task takes the cheaper kind (the static list gives pairs 0, 1, ...
// the tasks npairs, npairs + 1, ... next).  Chain: the layer-1 tiles of the
// first `lag` row blocks, then per row block k the layer-1 tiles of k and the
// layer-2 tiles of k - lag, then the rest of layer 2 (every layer-1 tile of a
// row block precedes that block's layer-2 tiles, and all CTAs are resident, so
// the row waits cannot form a cycle).
template <bool CHAIN>
__device__ __forceinline__ PairTask pair_decode(int q, const PairSched& sc) {
  PairTask t;
  if constexpr (!CHAIN) {
    t.layer = 0;
    const int nf = sc.L[0].n_dt - (sc.L[0].narrow ? 1 : 0);  // full tiles per row block
    if (q < sc.n_prow * nf) {
      t.prow = q / nf;
      t.dt = q % nf;
    } else {
      t.prow = q - sc.n_prow * nf;
      t.dt = nf;
    }
  } else {
    const int n1 = sc.L[0].n_dt, n2 = sc.L[1].n_dt;
    const int a = sc.lag * n1, per = n1 + n2, b = (sc.n_prow - sc.lag) * per;
    if (q < a) {
      t.layer = 0; t.prow = q / n1; t.dt = q % n1;
    } else if (q < a + b) {
      const int qq = q - a, k = sc.lag + qq / per, o = qq % per;
      if (o < n1) {
        t.layer = 0; t.prow = k; t.dt = o;
      } else {
        t.layer = 1; t.prow = k - sc.lag; t.dt = o - n1;
      }
    } else {
      const int qq = q - a - b;
      t.layer = 1; t.prow = sc.n_prow - sc.lag + qq / n2; t.dt = qq % n2;
    }
  }
  return t;
}

__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for a ring slot written by the leader (possibly from the other CTA).
__device__ __noinline__ bool ring_wait(uint64_t* b, uint32_t parity, int* abort_flag, int* status) {
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait_acq_cluster(b, parity)) {
    if (*(volatile int*)abort_flag) return false;
    if (gtimer() - t0 > kTimeoutNs) {
      *(volatile int*)abort_flag = 1;
      atomicExch(status, kErrTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// Bounded wait until a layer-1 row block is stored, then order the TMA loads
// that follow after the acquire.  Each of the block's `consumers` waiters then
// adds one; the last of them returns the counter to zero (nothing reads it
// again in this launch), so a launch leaves its counters zero without a pass
// over them at the end.
__device__ __noinline__ bool pair_wait_row(int* flag, int target, int consumers, int* abort_flag,
                                           int* status) {
  const uint64_t t0 = gtimer();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v >= target) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      if (atomicAdd(flag, 1) == target + consumers - 1) atomicExch(flag, 0);
      return true;
    }
    if (*(volatile int*)abort_flag) return false;
    if (gtimer() - t0 > kTimeoutNs) {
      *(volatile int*)abort_flag = 1;
      atomicExch(status, kErrTimeout);
      return false;
    }
    __nanosleep(256);
  }
}

// Task source of one role.  One layer: the static list.  Chain: the leader's
// producer (fetch = true) takes ids from the global counter and publishes them;
// every other role reads its CTA's ring and releases the slot on the leader.
template <bool CHAIN>
struct TaskSource {
  PairRing* ring;
  uint32_t leader_empty0;  // cluster address of the leader's ring empty[0]
  int* counter;
  uint32_t n;
  int next_static;
  int stride;
  // the leader's producer (one thread): take an id from the counter, publish it
  __device__ bool fetch(const PairSched& sc, int* id, int* abort_flag, int* status) {
    const int q = n % kPQ;
    const uint32_t ph = (n / kPQ) & 1;
    ++n;
    if (!wait_bounded(&ring->empty[q], ph ^ 1, abort_flag, status)) return false;
    const int v = atomicAdd(counter, 1);
    // every pair's leader stops at its first id past the end, so the counter's
    // last value is total + npairs - 1: that fetch returns it to zero
    if (v == sc.total + sc.npairs - 1) atomicExch(counter, 0);
    *id = v < sc.total ? v : -1;
    ring->id[q] = *id;
    const uint32_t peer_id = peer_addr(smem_u32(&ring->id[q]), 1);
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(peer_id), "r"(*id) : "memory");
    mbar_arrive(&ring->full[q]);
    arrive_remote(peer_addr(smem_u32(&ring->full[q]), 1));
    return true;
  }
  // one reading thread
  __device__ bool take1(const PairSched& sc, int* id, int* abort_flag, int* status) {
    if constexpr (!CHAIN) {
      *id = next_static < sc.total ? next_static : -1;
      next_static += stride;
      return true;
    } else {
      const int q = n % kPQ;
      const uint32_t ph = (n / kPQ) & 1;
      ++n;
      if (!ring_wait(&ring->full[q], ph, abort_flag, status)) return false;
      *id = *(volatile int*)&ring->id[q];
      arrive_remote(leader_empty0 + (uint32_t)(q * sizeof(uint64_t)));
      return true;
    }
  }
  // a whole warp: lane 0 waits and releases, every lane gets the id
  __device__ bool takew(const PairSched& sc, int lane, int* id, int* abort_flag, int* status) {
    if constexpr (!CHAIN) {
      *id = next_static < sc.total ? next_static : -1;
      next_static += stride;
      return true;
    } else {
      int ok = 1, v = -1;
      if (lane == 0) {
        ok = take1(sc, &v, abort_flag, status) ? 1 : 0;
      } else {
        ++n;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      v = __shfl_sync(0xffffffffu, v, 0);
      *id = v;
      return ok != 0;
    }
  }
};

// The epilogue of one tile for one warp: TMEM lane quarter q (rows row0 ..
// row0+31), out-channels dbase .. dbase+63 of a 128-channel tile.
template <int IO, int ACT, class Store>
__device__ __forceinline__ void pair_epilogue(uint32_t lane_addr, int ch, int lane, uint8_t* stg,
                                              uint32_t stg_s, const __half* bsm, int dbase,
                                              int Cout, uint32_t acc_empty_leader,
                                              const Store& store) {
  if (dbase >= Cout) {
    // the narrow last tile: this warp's 64 columns hold no output channel
    tc_fence_before();
    __syncwarp();
    if (lane == 0) arrive_remote_relaxed(acc_empty_leader);
    return;
  }
  // read the whole tile share out of TMEM: slices 0-1 into staging, 2-7 held;
  // each slice's TMEM load is issued before the previous slice is computed, so
  // one wait::ld covers it while that computation runs
  uint4 held[3][2][4];
  {
    const int cb = (PR_BD / 2) * ch;
    uint32_t va[4][8], vb[4][8];
    slice_load(lane_addr, cb, va);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t(&cur)[4][8] = (k & 1) ? vb : va;
      uint32_t(&nxt)[4][8] = (k & 1) ? va : vb;
      if (k < 7) slice_load(lane_addr, cb + 8 * (k + 1), nxt);
      uint4 o[4];
      slice_compute<IO, ACT>(cur, bsm + 8 * k, o);
      if (k < 2) {
        if (k == 0) {
          if (lane == 0) bulk_wait_read_all();  // the previous tile's last store read stg
          __syncwarp();
        }
        if constexpr (IO == kIoSpectralOut) {
          const int sw = (lane >> 2) & 1;
#pragma unroll
          for (int p = 0; p < 4; ++p)
            *reinterpret_cast<uint4*>(stg + p * 1024 + lane * 32 + ((k ^ sw) << 4)) = o[p];
        } else {
#pragma unroll
          for (int m = 0; m < 4; ++m)
            *reinterpret_cast<uint4*>(stg + lane * 128 + (((4 * k + m) ^ (lane & 7)) << 4)) = o[m];
        }
      } else {
#pragma unroll
        for (int m = 0; m < 4; ++m) held[(k - 2) >> 1][k & 1][m] = o[m];
      }
      if (k < 7) tmem_wait_ld();
    }
  }
  // TMEM is free for the next tile's MMAs once every warp of both CTAs got here.
  // The arrive is relaxed: what it hands back is TMEM, and every TMEM load of this
  // warp has completed (tcgen05.wait::ld) before it, so no memory operation needs
  // to be released with it; a release at cluster scope would first wait for this
  // thread's outstanding global writes (measured: about 0.6 us per tile).
  tc_fence_before();
  __syncwarp();
  if (lane == 0) arrive_remote_relaxed(acc_empty_leader);
  // stores: 16 out-channels x 32 rows each, while the next tile's MMAs run
#pragma unroll
  for (int sc = 0; sc < 4; ++sc) {
    const int d0 = dbase + 16 * sc;
    if (sc > 0) {
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      stage_two<IO>(stg, lane, held[sc - 1][0], held[sc - 1][1]);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0 && d0 < Cout) {
      store(stg_s, d0);
      bulk_commit();
    }
  }
}

// CHAIN = 0: one layer, output IO1 with ACT1.  CHAIN = 1: layer 1 writes H as
// tiled planes with ACT1, layer 2 writes Y spatially; `sync` = [next task,
// unused, one counter per row block], zero at launch and left zero (the last
// fetch of the task counter and the last waiter on a row counter reset them).
//
// Launched as a programmatic dependent of the previous kernel in the stream:
// the prologue (barriers, TMEM allocation) overlaps that kernel's last wave,
// and griddepcontrol.wait, which returns once that kernel has completed and
// its writes are visible, comes before the first global-memory access.
template <int ACT1, int IO1, int CHAIN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PR_THREADS, 1)
    eq_pair_tc_kernel(const __grid_constant__ CUtensorMap map_x1,
                      const __grid_constant__ CUtensorMap map_w1,
                      const __grid_constant__ CUtensorMap map_o1,
                      const __grid_constant__ CUtensorMap map_x2,
                      const __grid_constant__ CUtensorMap map_w2,
                      const __grid_constant__ CUtensorMap map_o2, PairSched sc, int* sync,
                      int* status) {
  static_assert(!CHAIN || IO1 == kIoSpectralOut, "a chain passes H as tiled planes");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PairBars* bars = reinterpret_cast<PairBars*>(smem + PR_OFF_BAR);
  PairRing* ring = reinterpret_cast<PairRing*>(smem + PR_OFF_BAR + sizeof(PairBars));
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cta_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PR_ST; ++s) {
      mbar_init(&bars->full[s], 1);   // the leader's producer arrives (with both CTAs' bytes)
      mbar_init(&bars->empty[s], 2);  // a multicast commit from each issuer
    }
    mbar_init(&bars->acc_full, 2);
    mbar_init(&bars->acc_empty, 2 * kEpiWarps);  // one arrival per epilogue warp of each CTA
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    for (int q = 0; q < kPQ; ++q) {
      mbar_init(&ring->full[q], 1);
      mbar_init(&ring->empty[q], kPRingReaders);
    }
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA completion
  tc_fence_after();
  grid_dependency_wait();
  const uint32_t tmem = bars->tmem_base;
  TaskSource<CHAIN> src{ring, peer_addr(smem_u32(&ring->empty[0]), 0), sync, 0u, pair, npairs};

  if (warp == 0) {
    // ---------------- producer: planes and this CTA's half of the weights ----------------
    if (lane == 0) {
      int issued_phase[PR_ST];
      for (int s = 0; s < PR_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      while (ok) {
        int id;
        if (CHAIN && rank == 0)
          ok = src.fetch(sc, &id, abort_flag, status);
        else
          ok = src.take1(sc, &id, abort_flag, status);
        if (!ok || id < 0) break;
        const PairTask t = pair_decode<CHAIN>(id, sc);
        const PairLayer& L = sc.L[t.layer];
        const CUtensorMap* mx = t.layer ? &map_x2 : &map_x1;
        const CUtensorMap* mw = t.layer ? &map_w2 : &map_w1;
        const int row = t.prow * 256 + 128 * (int)rank;
        if (CHAIN && t.layer == 1 &&
            !(ok = pair_wait_row(&sync[2 + t.prow], sc.flag_target, 2 * sc.L[1].n_dt,
                                 abort_flag, status)))
          break;
        for (int ks = 0; ks < L.n_ks; ++ks, ++it) {
          const int s = it % PR_ST;
          const uint32_t ph = (it / PR_ST) & 1;
          if (!(ok = wait_bounded(&bars->empty[s], ph ^ 1, abort_flag, status))) break;
          const uint32_t full_leader = peer_addr(smem_u32(&bars->full[s]), 0);
          const bool nar = pair_narrow(L, t.dt);
          if (rank == 0)
            mbar_expect_tx(&bars->full[s], 2 * (PR_XBYTES + (nar ? PR_WBYTES / 2 : PR_WBYTES)));
          const uint32_t slot = sbase + s * PR_STAGE;
          // planes: lines row/4 .. +32 of channel blocks 2ks, 2ks+1, all four planes
          tma_load_4d_pair(slot, mx, full_leader, 0, row / 4, PR_KSS * ks, 0);
          // this CTA's weight rows of the stage, boxes of 64 lines (8 KB)
          if (nar) {
            const int wline = L.narrow_line0 + (ks * 2 + (int)rank) * (PR_WLINES / 2);
            tma_load_2d_pair(slot + PR_XBYTES, mw, full_leader, 0, wline);
          } else {
            const int wline = ((t.dt * L.n_ks + ks) * 2 + (int)rank) * PR_WLINES;
            tma_load_2d_pair(slot + PR_XBYTES, mw, full_leader, 0, wline);
            tma_load_2d_pair(slot + PR_XBYTES + PR_WBYTES / 2, mw, full_leader, 0,
                             wline + PR_WLINES / 2);
          }
          issued_phase[s] = (int)ph;
        }
      }
      if (!ok && rank == 0) {
        // wait (bounded) for the loads this CTA pair put in flight on the leader's barriers
        for (int s = 0; s < PR_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->full[s], (uint32_t)issued_phase[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    // ---------------- MMA issuers (leader CTA): two threads, three products each ----------------
    // issuer 0 (warp 1): Y0 and Y1r; issuer 1 (warp 3): Y2 and Y1i.  Each commits
    // its own MMAs to the stage and tile barriers (two arrivals each), so the
    // ~70 cycles a tcgen05.mma costs its issuing thread are paid twice in parallel.
    if (rank == 0 && lane == 0) {
      const int who = warp == 1 ? 0 : 1;
      const uint32_t id_full = idesc_f16(256, PR_BD), id_full_neg = idesc_f16(256, PR_BD, true);
      const uint32_t id_nar = idesc_f16(256, PR_BD / 2), id_nar_neg = idesc_f16(256, PR_BD / 2, true);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      while (ok) {
        int id;
        if (!(ok = src.take1(sc, &id, abort_flag, status)) || id < 0) break;
        const PairTask t = pair_decode<CHAIN>(id, sc);
        const int n_ks = sc.L[t.layer].n_ks;
        // a narrow tile: N = 64, this CTA's 32 rows per weight plane
        const bool nar = pair_narrow(sc.L[t.layer], t.dt);
        const uint32_t id_n1 = nar ? id_nar : id_full, id_neg = nar ? id_nar_neg : id_full_neg;
        const uint32_t w_kstep = nar ? PR_WKS / 2 : PR_WKS;
        const uint32_t w_plane = nar ? 32 * PR_ROWB : 64 * PR_ROWB;
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < n_ks; ++ks, ++it) {
          const int s = it % PR_ST;
          if (!(ok = wait_bounded(&bars->full[s], (it / PR_ST) & 1, abort_flag, status))) break;
          tc_fence_after();
          const uint32_t xs = sbase + s * PR_STAGE, ws = xs + PR_XBYTES;
#pragma unroll
          for (int kk = 0; kk < PR_KSS; ++kk) {
            const uint32_t xa = xs + kk * PR_XBLK, wb = ws + kk * w_kstep;
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            const uint64_t xr = desc_kmajor<32>(xa + 2 * PR_XPLANE);
            const uint64_t xi = desc_kmajor<32>(xa + 3 * PR_XPLANE);
            const uint64_t br = desc_kmajor<32>(wb + 2 * w_plane);
            const uint64_t bi = desc_kmajor<32>(wb + 3 * w_plane);
            if (who == 0) {
              umma_pair(tmem + 0, desc_kmajor<32>(xa + 0 * PR_XPLANE),
                        desc_kmajor<32>(wb), id_n1, acc);                           // Y0
              umma_pair(tmem + 2 * PR_BD, xr, br, id_n1, acc);                      // Y1r
              umma_pair(tmem + 2 * PR_BD, xi, bi, id_neg, 1u);                      // -Xi Bi
            } else {
              umma_pair(tmem + PR_BD, desc_kmajor<32>(xa + 1 * PR_XPLANE),
                        desc_kmajor<32>(wb + w_plane), id_n1, acc);                 // Y2
              umma_pair(tmem + 3 * PR_BD, xr, bi, id_n1, acc);                      // Y1i
              umma_pair(tmem + 3 * PR_BD, xi, br, id_n1, 1u);
            }
          }
          umma_commit_pair(&bars->empty[s], 3);
        }
        if (ok) umma_commit_pair(&bars->acc_full, 3);
        ++tcount;
      }
      // every MMA this thread issued completes before TMEM is freed
      umma_commit_pair(&bars->drain[who], 1);
      drain_wait(&bars->drain[who], 0);
    }
    __syncwarp();
  } else if (warp >= PR_EPI0 && warp < PR_EPI0 + kEpiWarps) {
    // ---------------- epilogue (both CTAs, own rows) ----------------
    const int q = warp & 3;               // TMEM lane quarter = rows 32q..32q+31
    const int ch = (warp - PR_EPI0) >> 2;  // out-channel half of the tile
    uint8_t* stg = smem + PR_OFF_STG + (warp - PR_EPI0) * kStgBytes;
    const uint32_t stg_s = smem_u32(stg);
    __half* bsm = reinterpret_cast<__half*>(smem + PR_OFF_BIAS + (warp - PR_EPI0) * 128);
    const uint32_t acc_empty_leader = peer_addr(smem_u32(&bars->acc_empty), 0);
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
    uint32_t tcount = 0;
    while (true) {
      int id;
      if (!src.takew(sc, lane, &id, abort_flag, status) || id < 0) break;
      const PairTask t = pair_decode<CHAIN>(id, sc);
      const PairLayer& L = sc.L[t.layer];
      const int64_t row0 = (int64_t)t.prow * 256 + 128 * rank + 32 * q;
      const int dbase = t.dt * PR_BD + (PR_BD / 2) * ch;
      if (2 * lane < PR_BD / 2) {
        const int d = dbase + 2 * lane;
        uint32_t v = 0u;
        if (L.bias && d < L.Cout) v = *reinterpret_cast<const uint32_t*>(L.bias + d);  // Cout even
        reinterpret_cast<uint32_t*>(bsm)[lane] = v;
      }
      __syncwarp();
      if (!warp_wait(&bars->acc_full, tcount & 1, abort_flag, status)) break;
      tc_fence_after();
      if (t.layer == 0) {
        pair_epilogue<IO1, ACT1>(lane_addr, ch, lane, stg, stg_s, bsm, dbase, L.Cout,
                                 acc_empty_leader, PairStoreOf<IO1>{&map_o1, row0, sc.N});
      } else if constexpr (CHAIN) {
        pair_epilogue<kIoSpatial, 0>(lane_addr, ch, lane, stg, stg_s, bsm, dbase, L.Cout,
                                     acc_empty_leader, RowStore<4>{&map_o2, row0, sc.N});
      }
      ++tcount;
      if (CHAIN && t.layer == 0) {
        // this warp's part of the H tile is in memory: count it for the row block
        if (lane == 0) {
          bulk_wait_all();
          asm volatile("fence.proxy.async.global;" ::: "memory");
          asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(&sync[2 + t.prow])
                       : "memory");
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  grid_launch_dependents();  // this CTA has no more work: the next kernel may launch
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// Prepared planes [P][Cout][Cin] (P = 5 at T = 4: A0, A2, Br, Bi, -Bi) -> the
// pair kernel's weight stages.  A 128-channel tile: blob (dt, stage, rank) =
// two K steps (channels 32*stage + 16*kk ..+16) of 256 rows x 16 channels (32
// bytes, 32-byte swizzle: 16-byte piece ^= (row / 4) % 2); rows 64j .. 64j+63
// hold plane j (A0, A2, Br, Bi) at out-channels dt*128 + 64*rank + (row % 64).
// The narrow last tile (<= 64 channels, after the full ones): blob (stage,
// rank) = two K steps of 128 rows, rows 32j .. 32j+31 = plane j at out-channels
// dt*128 + 32*rank + (row % 32).  Zero past the matrix.  One thread per 16-byte
// piece.
__global__ void pair_tile_weights_kernel(const __half* __restrict__ planes, int Cin, int Cout,
                                         int n_ks, int n_full, int64_t n_pieces,
                                         uint4* __restrict__ tiles) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pieces) return;
  const int64_t full_pieces = (int64_t)n_full * n_ks * 2 * (PR_WBYTES / 16);
  const bool nar = idx >= full_pieces;
  const int64_t j = nar ? idx - full_pieces : idx;
  const int rows = nar ? PR_WROWS / 2 : PR_WROWS;  // rows of one K step of a blob
  const int piece = (int)(j & 1);
  const int r = (int)((j >> 1) % rows);
  const int64_t kblob = (j >> 1) / rows;  // (dt, stage, rank, kk), narrow: (stage, rank, kk)
  const int kk = (int)(kblob % PR_KSS);
  const int64_t blob = kblob / PR_KSS;
  const int rank = (int)(blob & 1);
  const int64_t dk = blob >> 1;
  const int dt = nar ? n_full : (int)(dk / n_ks);
  const int ks = (int)(dk % n_ks) * PR_KSS + kk;
  const int per = rows / 4;  // rows per plane
  const int plane = r / per;
  const int d = dt * PR_BD + per * rank + (r % per);
  const int c0 = ks * PR_KC + piece * 8;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (d < Cout && c0 < Cin)  // Cin % 16 == 0: the 8 channels are all in range
    v = *reinterpret_cast<const uint4*>(planes + ((int64_t)plane * Cout + d) * Cin + c0);
  const int64_t base = nar ? full_pieces * 16 : 0;
  const int64_t dst = base + kblob * (rows * PR_ROWB) + r * PR_ROWB + ((piece ^ ((r >> 2) & 1)) << 4);
  tiles[dst >> 4] = v;
}

// Group DFT of p4 rows into tiled planes (layout above): X [N][C*4] -> the
// four planes, each value times 1/4 (FP32 arithmetic, one rounding), rows
// N..Np-1 zero.  A thread takes 8 channels of one row (64 bytes of X, four
// 16-byte loads) and writes one 16-byte half row per plane; a warp takes 16
// rows of one 16-channel block (lane l: row l/2, channels 8(l%2)..+7), so each
// of its four plane stores fills 512 contiguous bytes of the tiled layout.
__global__ void group_dft_tiled_kernel(const uint4* __restrict__ X, int64_t N, int64_t Np, int C,
                                       uint8_t* __restrict__ out) {
  grid_dependency_wait();
  grid_launch_dependents();
  const int KB = C / 16;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= Np / 16 * KB) return;
  const int lane = (int)(threadIdx.x & 31);
  const int kb = (int)(w % KB), h = lane & 1;
  const int64_t n = (w / KB) * 16 + (lane >> 1);
  uint4 v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[k] = make_uint4(0u, 0u, 0u, 0u);
    if (n < N) v[k] = X[(n * C * 8 + (int64_t)kb * 128 + h * 64) / 16 + k];
  }
  uint32_t o[4][4];  // [plane][channel pair k]: channels 8h + 2k, 8h + 2k + 1
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t w4[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    float f0[2], fh[2], fr[2], fi[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {  // channel 8h + 2k + e: x0 x1 | x2 x3
      const float2 lo = unpack_h2(w4[2 * e]), hi = unpack_h2(w4[2 * e + 1]);
      const float x0 = lo.x, x1 = lo.y, x2 = hi.x, x3 = hi.y;
      const float a = x0 + x2, b = x1 + x3;
      f0[e] = (a + b) * 0.25f;
      fh[e] = (a - b) * 0.25f;
      fr[e] = (x0 - x2) * 0.25f;
      fi[e] = (x3 - x1) * 0.25f;
    }
    o[0][k] = pack_h2(f0[0], f0[1]);
    o[1][k] = pack_h2(fh[0], fh[1]);
    o[2][k] = pack_h2(fr[0], fr[1]);
    o[3][k] = pack_h2(fi[0], fi[1]);
  }
  const int64_t inrow = n * 32 + ((h ^ (int)((n >> 2) & 1)) << 4);
#pragma unroll
  for (int p = 0; p < 4; ++p)
    *reinterpret_cast<uint4*>(out + ((int64_t)p * KB + kb) * Np * 32 + inrow) =
        make_uint4(o[p][0], o[p][1], o[p][2], o[p][3]);
}

// 4-D view of tiled planes: (64 halves of a 128-byte line, Np/4 lines of a
// channel block, C/16 blocks, 4 planes); box = `lines` lines x `blocks` blocks x
// all 4 planes, landing as [plane][block][line][128 B].
bool encode_tiled_map(CUtensorMap* m, const void* base, int channels, int64_t Np, uint32_t lines,
                      uint32_t blocks) {
  auto encode = encode_fn();
  cuuint64_t dims[4] = {64, (cuuint64_t)(Np / 4), (cuuint64_t)(channels / 16), 4};
  cuuint64_t strides[3] = {128, (cuuint64_t)Np * 32, (cuuint64_t)Np * 32 * (channels / 16)};
  cuuint32_t box[4] = {64, lines, blocks, 4};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int ACT, int IO, int CHAIN>
cudaError_t set_pair_attr() {
  return cudaFuncSetAttribute(eq_pair_tc_kernel<ACT, IO, CHAIN>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, PR_SMEM);
}

// The weight stages as 128-byte lines, copied verbatim (already swizzled).
bool encode_pair_weights(CUtensorMap* m, const void* tiles, int Cin, int Cout);
// Y [N][Cout*4] spatial: store box = 1 chunk of 128 B x 32 rows.
bool encode_rows_store(CUtensorMap* m, void* Y, int Cout, int64_t N);

// Co-resident pairs (a cluster must fit inside one GPC, so this can be below
// num_sms / 2); every variant has the same resources, so one query serves all.
int pair_capacity(const void* kernel, int num_sms) {
  static int max_pairs = 0;
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)(num_sms / 2));
    cfg.blockDim = dim3(PR_THREADS);
    cfg.dynamicSmemBytes = PR_SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    max_pairs = n < num_sms / 2 ? n : num_sms / 2;
  }
  return max_pairs;
}

cudaError_t set_all_pair_attrs() {
  static bool done = false;
  if (done) return cudaSuccess;
  cudaError_t e = set_pair_attr<0, kIoSpatial, 0>();
  if (e == cudaSuccess) e = set_pair_attr<1, kIoSpatial, 0>();
  if (e == cudaSuccess) e = set_pair_attr<0, kIoSpectralOut, 0>();
  if (e == cudaSuccess) e = set_pair_attr<1, kIoSpectralOut, 0>();
  if (e == cudaSuccess) e = set_pair_attr<0, kIoSpectralOut, 1>();
  if (e == cudaSuccess) e = set_pair_attr<1, kIoSpectralOut, 1>();
  if (e == cudaSuccess) done = true;
  return e;
}

}  // namespace

int64_t tiled_rows(int64_t N) { return (N + 127) / 128 * 128; }

size_t tiled_planes_bytes(int64_t N, int channels) {
  return (size_t)4 * (size_t)tiled_rows(N) * (size_t)channels * 2;
}

cudaError_t launch_group_dft_tiled(const void* X, int64_t N, int C, void* out, cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  if (C % 16 != 0) return cudaErrorInvalidValue;
  const int64_t Np = tiled_rows(N);
  const int64_t threads = Np / 16 * (C / 16) * 32;
  return launch_dependent(group_dft_tiled_kernel, dim3((unsigned)((threads + 255) / 256)),
                          dim3(256), 0, st, static_cast<const uint4*>(X), N, Np, C,
                          static_cast<uint8_t*>(out));
}

bool pair_tc_supported(int64_t N, int Cin, int Cout) {
  return N >= 1 && N <= 0x7fffff00LL && Cin % 16 == 0 && Cout % 16 == 0 && Cin >= 16 &&
         Cout >= 16;
}

namespace {
// out-channel tiles of a layer: full 128-channel tiles, then a narrow one when
// the remainder is at most 64 channels
int pair_n_dt(int Cout) { return (Cout + PR_BD - 1) / PR_BD; }
bool pair_has_narrow(int Cout) { return Cout - (pair_n_dt(Cout) - 1) * PR_BD <= PR_BD / 2; }
int pair_n_ks(int Cin) { return (Cin + PR_KC * PR_KSS - 1) / (PR_KC * PR_KSS); }
}  // namespace

size_t pair_tile_bytes(int Cin, int Cout) {
  const size_t n_st = (size_t)pair_n_ks(Cin);
  const size_t nar = pair_has_narrow(Cout) ? 1 : 0, n_full = (size_t)pair_n_dt(Cout) - nar;
  return n_full * n_st * 2 * PR_WBYTES + nar * n_st * 2 * (PR_WBYTES / 2);
}

cudaError_t launch_pair_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                     cudaStream_t st) {
  const int n_ks = pair_n_ks(Cin);
  const int n_full = pair_n_dt(Cout) - (pair_has_narrow(Cout) ? 1 : 0);
  const int64_t n_pieces = (int64_t)pair_tile_bytes(Cin, Cout) / 16;
  pair_tile_weights_kernel<<<(unsigned)((n_pieces + 255) / 256), 256, 0, st>>>(
      static_cast<const __half*>(planes), Cin, Cout, n_ks, n_full, n_pieces,
      static_cast<uint4*>(tiles));
  return cudaGetLastError();
}

namespace {

bool encode_pair_weights(CUtensorMap* m, const void* tiles, int Cin, int Cout) {
  auto encode = encode_fn();
  const uint64_t lines = pair_tile_bytes(Cin, Cout) / 128;
  cuuint64_t dims[2] = {64, (cuuint64_t)lines};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, PR_WLINES / 2};
  cuuint32_t estr[2] = {1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(tiles), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_rows_store(CUtensorMap* m, void* Y, int Cout, int64_t N) {
  auto encode = encode_fn();
  cuuint64_t ydims[3] = {64, (cuuint64_t)Cout * 4 / 64, (cuuint64_t)N};
  cuuint64_t ystrides[2] = {128, (cuuint64_t)Cout * 4 * 2};
  cuuint32_t ybox[3] = {64, 1, 32};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, Y, ydims, ystrides, ybox, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

PairLayer pair_layer(int Cin, int Cout, const void* bias) {
  PairLayer L;
  L.n_dt = pair_n_dt(Cout);
  L.n_ks = pair_n_ks(Cin);  // a last half stage reads zeros
  L.Cout = Cout;
  L.narrow = pair_has_narrow(Cout) ? 1 : 0;
  L.narrow_line0 = (L.n_dt - L.narrow) * L.n_ks * 2 * PR_WLINES;
  L.bias = static_cast<const __half*>(bias);
  return L;
}

}  // namespace

cudaError_t launch_pair_tc(const void* Xt, int64_t N, int Cin, int Cout, const void* tiles,
                           const void* bias, void* Y, int* status, int num_sms, int act,
                           int spectral_out, cudaStream_t st) {
  if (!pair_tc_supported(N, Cin, Cout) || !tiles) return cudaErrorNotSupported;
  if (act != 0 && act != 1) return cudaErrorInvalidValue;
  if (!encode_fn()) return cudaErrorNotSupported;
  CUtensorMap mx, mw, my;
  const int64_t Np = tiled_rows(N);
  // input planes (tiled): box = 32 lines (128 rows) x 2 channel blocks x 4 planes
  if (!encode_tiled_map(&mx, Xt, Cin, Np, 32, PR_KSS) || !encode_pair_weights(&mw, tiles, Cin, Cout))
    return cudaErrorInvalidValue;
  if (spectral_out) {
    // next layer's tiled planes: store box = 8 lines (32 rows) x 4 planes
    if (!encode_tiled_map(&my, Y, Cout, Np, 8, 1)) return cudaErrorInvalidValue;
  } else if (!encode_rows_store(&my, Y, Cout, N)) {
    return cudaErrorInvalidValue;
  }
  PairSched sc = {};
  sc.N = N;
  sc.n_prow = (int)((N + 255) / 256);
  sc.L[0] = pair_layer(Cin, Cout, bias);
  sc.L[1] = sc.L[0];
  if ((int64_t)sc.n_prow * sc.L[0].n_dt > 0x7fffffffLL) return cudaErrorInvalidValue;
  sc.total = sc.n_prow * sc.L[0].n_dt;
  cudaError_t e = set_all_pair_attrs();
  if (e != cudaSuccess) return e;
  auto kernel = act ? (spectral_out ? eq_pair_tc_kernel<1, kIoSpectralOut, 0>
                                    : eq_pair_tc_kernel<1, kIoSpatial, 0>)
                    : (spectral_out ? eq_pair_tc_kernel<0, kIoSpectralOut, 0>
                                    : eq_pair_tc_kernel<0, kIoSpatial, 0>);
  int npairs = pair_capacity((const void*)kernel, num_sms);
  if (npairs > sc.total) npairs = sc.total;
  return launch_dependent(kernel, dim3(2 * npairs), dim3(PR_THREADS), PR_SMEM, st, mx, mw, my, mx,
                          mw, my, sc, (int*)nullptr, status);
}

size_t pair_chain_sync_bytes(int64_t N) { return (size_t)(2 + (N + 255) / 256) * sizeof(int); }

cudaError_t launch_pair_chain_tc(const void* Xt, int64_t N, int C0, int C1, int C2,
                                 const void* W1tiles, const void* b1, const void* W2tiles,
                                 const void* b2, void* Ht, void* Y, int* sync, int* status,
                                 int num_sms, int act1, cudaStream_t st) {
  if (!pair_tc_supported(N, C0, C1) || !pair_tc_supported(N, C1, C2) || !W1tiles || !W2tiles)
    return cudaErrorNotSupported;
  if (act1 != 0 && act1 != 1) return cudaErrorInvalidValue;
  if (!encode_fn()) return cudaErrorNotSupported;
  const int64_t Np = tiled_rows(N);
  CUtensorMap mx1, mw1, mh_st, mh_ld, mw2, my;
  if (!encode_tiled_map(&mx1, Xt, C0, Np, 32, PR_KSS) ||
      !encode_pair_weights(&mw1, W1tiles, C0, C1) ||
      !encode_tiled_map(&mh_st, Ht, C1, Np, 8, 1) ||
      !encode_tiled_map(&mh_ld, Ht, C1, Np, 32, PR_KSS) ||
      !encode_pair_weights(&mw2, W2tiles, C1, C2) || !encode_rows_store(&my, Y, C2, N))
    return cudaErrorInvalidValue;
  PairSched sc = {};
  sc.N = N;
  sc.n_prow = (int)((N + 255) / 256);
  sc.L[0] = pair_layer(C0, C1, b1);
  sc.L[1] = pair_layer(C1, C2, b2);
  if ((int64_t)sc.n_prow * (sc.L[0].n_dt + sc.L[1].n_dt) > 0x7fffffffLL)
    return cudaErrorInvalidValue;
  sc.total = sc.n_prow * (sc.L[0].n_dt + sc.L[1].n_dt);
  cudaError_t e = set_all_pair_attrs();
  if (e != cudaSuccess) return e;
  auto kernel = act1 ? eq_pair_tc_kernel<1, kIoSpectralOut, 1> : eq_pair_tc_kernel<0, kIoSpectralOut, 1>;
  int npairs = pair_capacity((const void*)kernel, num_sms);
  if (npairs > sc.total) npairs = sc.total;
  // layer-1 row blocks queued ahead of layer 2: about 0.6 of the blocks, at least
  // a wave of layer-1 tiles
  const int wave = (npairs + sc.L[0].n_dt - 1) / sc.L[0].n_dt;
  int lag = (3 * sc.n_prow + 2) / 5;
  if (lag < wave) lag = wave;
  sc.lag = lag < sc.n_prow ? lag : sc.n_prow;
  sc.flag_target = 2 * kEpiWarps * sc.L[0].n_dt;
  sc.npairs = npairs;
  return launch_dependent(kernel, dim3(2 * npairs), dim3(PR_THREADS), PR_SMEM, st, mx1, mw1, mh_st,
                          mh_ld, mw2, my, sc, sync, status);
}

}  // namespace eql
