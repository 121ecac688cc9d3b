// tcgen05/TMEM tensor-core forward of the p4 (T = 4) EQ-Linear layer, FP16 in,
// FP32 accumulate, FP16 out, for sm_100a.
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" and
// "Specialisation for p4"): per row n and input channel c the group DFT
//   X0 = x0+x1+x2+x3,  X2 = x0-x1+x2-x3,  Xr = x0-x2,  Xi = x3-x1
// (adds only), six real GEMMs against the prepared weight planes
//   Y0 = X0 A0^T,  Y2 = X2 A2^T,  [Y1r | Y1i] = Xr [Br | Bi]^T + Xi [-Bi | Br]^T
// and the inverse DFT with the dyadic factors 1/4 and 1/2, plus bias:
//   y0 = (Y0+Y2)/4 + Y1r/2,  y1 = (Y0-Y2)/4 - Y1i/2,
//   y2 = (Y0+Y2)/4 - Y1r/2,  y3 = (Y0-Y2)/4 + Y1i/2.
//
// Design (one persistent CTA per SM, tile = 128 rows x BD out-channels):
//   warp 0      TMA producer: raw X tiles (128 rows x 32 channels x 4, two
//               128B-swizzled boxes) and the five weight planes of the stage.
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma (M=128, K=16).
//   warps 4-7   epilogue: tcgen05.ld of the four accumulators, inverse DFT,
//               bias, FP16 pack, 16-byte global stores (one row per thread).
//   warps 8-15  transform: group DFT of the raw tile in FP32, one rounding to
//               FP16, written as four K-major 64B-swizzled operand planes.
// The accumulators live in TMEM: Y0 at columns [0,BD), Y2 [BD,2BD),
// Y1r [2BD,3BD), Y1i [3BD,4BD).  The freq-1 B operand is the contiguous stack
// of planes [-Bi | Br | Bi] in shared memory: rows [BD,3BD) are [Br|Bi] and rows
// [0,2BD) are [-Bi|Br], so each complex product is one N = 2*BD MMA.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the CTA
// sets a shared abort flag and the plan's status word, drains what it issued and
// returns, so a stuck pipeline never hangs the GPU.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "eql_kernels.h"

namespace eql {
namespace {

constexpr int kT = 4;
constexpr int BM = 128;          // rows per tile = MMA M
constexpr int BD = 128;          // out-channels per tile
constexpr int BK = 16;           // in-channels per pipeline stage = one MMA K step
constexpr int RAW_ST = 5;        // raw X ring (covers HBM latency)
constexpr int PL_ST = 3;         // transformed operand ring
constexpr int W_ST = 4;          // weight-plane ring (L2-resident source)
constexpr int kPlanes = 5;       // A0, A2, -Bi, Br, Bi
constexpr int kThreads = 512;
constexpr int kEpiWarp0 = 4;
constexpr int kXfWarp0 = 8;
constexpr int kXfWarps = 8;
constexpr uint32_t kTmemCols = 4 * BD;  // 512

constexpr uint32_t RAW_STAGE_BYTES = BM * 128;            // 16 channels x 4 x 2 B per row
constexpr uint32_t PLANE_BYTES = BM * BK * 2;             // 128 rows x 32 B
constexpr uint32_t PL_STAGE_BYTES = 4 * PLANE_BYTES;
constexpr uint32_t WREG_BYTES = BD * BK * 2;              // BD rows x 32 B
constexpr uint32_t W_STAGE_BYTES = kPlanes * WREG_BYTES;
constexpr uint32_t OFF_RAW = 0;
constexpr uint32_t OFF_PL = OFF_RAW + RAW_ST * RAW_STAGE_BYTES;
constexpr uint32_t OFF_W = OFF_PL + PL_ST * PL_STAGE_BYTES;
constexpr uint32_t OFF_BAR = OFF_W + W_ST * W_STAGE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;     // barriers + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

constexpr unsigned long long kTimeoutNs = 2000000000ull;

// status word codes
constexpr int kErrTimeout = 1;

struct Bars {
  uint64_t raw_full[RAW_ST], raw_empty[RAW_ST];
  uint64_t pl_full[PL_ST], pl_empty[PL_ST];
  uint64_t w_full[W_ST], w_empty[W_ST];
  uint64_t acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false if the CTA aborted or the wait timed out (then aborts it).
__device__ __noinline__ bool wait_bounded(uint64_t* b, uint32_t parity, Bars* bars, int* status) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = gtimer();
  while (true) {
    if (mbar_try_wait(b, parity)) return true;
    if (*(volatile int*)&bars->abort_flag) return false;
    if (gtimer() - t0 > kTimeoutNs) {
      *(volatile int*)&bars->abort_flag = 1;
      atomicExch(status, kErrTimeout);
      return false;
    }
  }
}
// Warp-uniform bounded wait: every lane polls, then the warp agrees, so a lane
// that gave up cannot leave the others waiting at a warp-synchronous point.
__device__ __forceinline__ bool warp_wait(uint64_t* b, uint32_t parity, Bars* bars, int* status) {
  const bool ok = wait_bounded(b, parity, bars, status);
  return __all_sync(0xffffffffu, ok);
}
// Bounded wait used while draining after an abort (ignores the abort flag).
__device__ __noinline__ void drain_wait(uint64_t* b, uint32_t parity) {
  const uint64_t t0 = gtimer();
  while (!mbar_try_wait(b, parity)) {
    if (gtimer() - t0 > kTimeoutNs) return;
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// K-major, 32-byte-swizzled operand tile: rows of 32 B (16 fp16 of K = one MMA
// K step), 8-row groups 256 B apart (SBO), descriptor version 1 (sm_100),
// layout type 6 (SWIZZLE_32B: 16-byte chunk index ^= (row / 4) % 2).
__device__ __forceinline__ uint64_t desc_kmajor_sw32(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;              // leading byte offset (unused when swizzled)
  d |= (uint64_t)(256u >> 4) << 32;     // stride byte offset: 8 rows x 32 B
  d |= (uint64_t)1u << 46;              // descriptor version for sm_100
  d |= (uint64_t)6u << 61;              // SWIZZLE_32B
  return d;
}
// Instruction descriptor, kind::f16: A = B = F16, D = F32, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 TMEM lanes x 256 bits: thread t gets lanes (t/4) and (t/4 + 8) of the
// addressed 16-lane group, columns 2*(t%4) and 2*(t%4)+1 -> regs
// {lane t/4: col, col+1, lane t/4+8: col, col+1}.
#define EQL_TMEM_LD_16x256(taddr, r)                                                   \
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0, %1, %2, %3}, [%4];"         \
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])                         \
               : "r"(taddr))

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);  // a -> low half, b -> high half
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}
__device__ __forceinline__ float2 unpack_h2(uint32_t u) {
  __half2 h;
  memcpy(&h, &u, 4);
  return __half22float2(h);
}

struct TileInfo {
  int n_dt;       // d tiles
  int num_tiles;  // row tiles x d tiles
  int k_stages;   // ceil(Cin / BK)
};

__global__ void __launch_bounds__(kThreads, 1)
    p4_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_w, const __half* __restrict__ bias,
                     __half* __restrict__ Y, int64_t N, int Cin, int Cout, TileInfo ti,
                     int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled TMA destinations and operand tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RAW_ST; ++s) {
      mbar_init(&bars->raw_full[s], 1);
      mbar_init(&bars->raw_empty[s], kXfWarps);
    }
    for (int s = 0; s < PL_ST; ++s) {
      mbar_init(&bars->pl_full[s], kXfWarps);
      mbar_init(&bars->pl_empty[s], 1);
    }
    for (int s = 0; s < W_ST; ++s) {
      mbar_init(&bars->w_full[s], 1);
      mbar_init(&bars->w_empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 4 * 32);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 || warp == 2) {
    // ---------------- TMA producers: warp 0 raw X, warp 2 weight planes ----------------
    if (lane == 0) {
      const bool is_raw = (warp == 0);
      const int depth = is_raw ? RAW_ST : W_ST;
      uint64_t* full = is_raw ? bars->raw_full : bars->w_full;
      uint64_t* empty = is_raw ? bars->raw_empty : bars->w_empty;
      int issued_phase[RAW_ST > W_ST ? RAW_ST : W_ST];  // last phase issued per slot
      for (int s = 0; s < depth; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      // smem regions: 0 = A0, 1 = A2, 2 = -Bi, 3 = Br, 4 = Bi (prepared planes 0,1,4,2,3)
      const int src_plane[kPlanes] = {0, 1, 4, 2, 3};
      for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x) {
        const int row0 = (tile / ti.n_dt) * BM;
        const int d0 = (tile % ti.n_dt) * BD;
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int s = it % depth;
          const uint32_t ph = (it / depth) & 1;
          const int c0 = ks * BK;
          if (!(ok = wait_bounded(&empty[s], ph ^ 1, bars, status))) break;
          if (is_raw) {
            mbar_expect_tx(&full[s], RAW_STAGE_BYTES);
            tma_load_2d(sbase + OFF_RAW + s * RAW_STAGE_BYTES, &map_x, &full[s], c0 * kT, row0);
          } else {
            mbar_expect_tx(&full[s], W_STAGE_BYTES);
            const uint32_t wdst = sbase + OFF_W + s * W_STAGE_BYTES;
#pragma unroll
            for (int r = 0; r < kPlanes; ++r)
              tma_load_3d(wdst + r * WREG_BYTES, &map_w, &full[s], c0, d0, src_plane[r]);
          }
          issued_phase[s] = (int)ph;
        }
      }
      if (!ok) {
        // wait (bounded) for the copies this thread put in flight
        for (int s = 0; s < depth; ++s)
          if (issued_phase[s] >= 0) drain_wait(&full[s], (uint32_t)issued_phase[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const uint32_t id_n1 = idesc_f16(BM, BD);
      const uint32_t id_n2 = idesc_f16(BM, 2 * BD);
      for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x, ++tcount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, bars, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int sp = it % PL_ST, sw = it % W_ST;
          if (!(ok = wait_bounded(&bars->pl_full[sp], (it / PL_ST) & 1, bars, status))) break;
          if (!(ok = wait_bounded(&bars->w_full[sw], (it / W_ST) & 1, bars, status))) break;
          tc_fence_after();
          const uint32_t pl = sbase + OFF_PL + sp * PL_STAGE_BYTES;
          const uint32_t wr = sbase + OFF_W + sw * W_STAGE_BYTES;
          const uint32_t acc = ks > 0 ? 1u : 0u;
          // Y0 += X0 A0^T ; Y2 += X2 A2^T ; [Y1r|Y1i] += Xr [Br|Bi]^T + Xi [-Bi|Br]^T
          umma(tmem + 0, desc_kmajor_sw32(pl + 0 * PLANE_BYTES),
               desc_kmajor_sw32(wr + 0 * WREG_BYTES), id_n1, acc);
          umma(tmem + BD, desc_kmajor_sw32(pl + 1 * PLANE_BYTES),
               desc_kmajor_sw32(wr + 1 * WREG_BYTES), id_n1, acc);
          umma(tmem + 2 * BD, desc_kmajor_sw32(pl + 2 * PLANE_BYTES),
               desc_kmajor_sw32(wr + 3 * WREG_BYTES), id_n2, acc);
          umma(tmem + 2 * BD, desc_kmajor_sw32(pl + 3 * PLANE_BYTES),
               desc_kmajor_sw32(wr + 2 * WREG_BYTES), id_n2, 1u);
          umma_commit(&bars->pl_empty[sp]);
          umma_commit(&bars->w_empty[sw]);
        }
        if (ok) umma_commit(&bars->acc_full);
      }
      // all MMAs this thread issued must be complete before TMEM is freed
      umma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ---------------- epilogue ----------------
    const int q = warp - kEpiWarp0;  // TMEM lane quarter: rows 32q .. 32q+31
    uint32_t tcount = 0;
    const int64_t ldy = (int64_t)Cout * kT;
    const int tr = lane >> 2, tc = 2 * (lane & 3);  // row-in-8 and column pair of this lane
    for (int tile = blockIdx.x; tile < ti.num_tiles; tile += gridDim.x, ++tcount) {
      if (!warp_wait(&bars->acc_full, tcount & 1, bars, status)) break;
      tc_fence_after();
      const int64_t rbase = (int64_t)(tile / ti.n_dt) * BM + 32 * q;
      const int d0 = (tile % ti.n_dt) * BD;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {  // 16-lane halves of the quarter
        const uint32_t laddr = tmem + ((uint32_t)(32 * q + 16 * h) << 16);
        const int64_t row_a = rbase + 16 * h + tr, row_b = row_a + 8;
#pragma unroll 2
        for (int dc = 0; dc < BD; dc += 8) {
          uint32_t a0[4], a2[4], ar[4], ai[4];
          EQL_TMEM_LD_16x256(laddr + dc, a0);
          EQL_TMEM_LD_16x256(laddr + BD + dc, a2);
          EQL_TMEM_LD_16x256(laddr + 2 * BD + dc, ar);
          EQL_TMEM_LD_16x256(laddr + 3 * BD + dc, ai);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          const int d = d0 + dc + tc;  // this lane's two out-channels: d, d+1
          if (d >= Cout) continue;
          float b0 = 0.f, b1 = 0.f;
          if (bias) {
            const float2 bb = __half22float2(*reinterpret_cast<const __half2*>(bias + d));
            b0 = bb.x;
            b1 = bb.y;
          }
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {  // reg pair rr: row_a (rr=0) or row_b (rr=1)
            const int64_t row = rr ? row_b : row_a;
            if (row >= N) continue;
            uint32_t packed[4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {  // out-channel d + hh
              const int k = 2 * rr + hh;
              const float y0 = __uint_as_float(a0[k]), y2 = __uint_as_float(a2[k]);
              const float yr = __uint_as_float(ar[k]), yi = __uint_as_float(ai[k]);
              const float b = hh ? b1 : b0;
              const float e = (y0 + y2) * 0.25f, o = (y0 - y2) * 0.25f;
              const float r = yr * 0.5f, m = yi * 0.5f;
              packed[2 * hh + 0] = pack_h2(e + r + b, o - m + b);
              packed[2 * hh + 1] = pack_h2(e - r + b, o + m + b);
            }
            *reinterpret_cast<uint4*>(Y + row * ldy + (int64_t)d * kT) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
  } else if (warp >= kXfWarp0) {
    // ---------------- transform: group DFT into the operand planes ----------------
    // One unit = one row x 8 channels: four 16-byte raw chunks in, one 16-byte
    // chunk out per plane.  Lanes take consecutive rows, so the swizzled raw
    // reads and plane writes of each 8-lane phase hit distinct banks.
    const int xt = threadIdx.x - kXfWarp0 * 32;  // 0..255
    const int r = xt & (BM - 1);                 // row of the tile
    const int qc = xt >> 7;                      // 8-channel half of the stage (0, 1)
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x) {
      for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
        const int sr = it % RAW_ST, sp = it % PL_ST;
        if (!(ok = warp_wait(&bars->raw_full[sr], (it / RAW_ST) & 1, bars, status))) break;
        if (!(ok = warp_wait(&bars->pl_empty[sp], ((it / PL_ST) & 1) ^ 1, bars, status))) break;
        // raw: row r is 128 B (16 channels x 4), 16 B chunk j at (j ^ (r % 8)) * 16
        const uint8_t* rb = smem + OFF_RAW + sr * RAW_STAGE_BYTES + r * 128;
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = qc * 4 + i;
          v[i] = *reinterpret_cast<const uint4*>(rb + ((j ^ (r & 7)) << 4));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->raw_empty[sr]);
        // chunk i holds channels 2i (.x = x0,x1  .y = x2,x3) and 2i+1 (.z, .w)
        uint32_t o0[4], o2[4], orr[4], oi[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float f0[2], f2[2], fr[2], fi[2];
          const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const float2 lo = unpack_h2(w4[2 * hh]), hi = unpack_h2(w4[2 * hh + 1]);
            const float x0 = lo.x, x1 = lo.y, x2 = hi.x, x3 = hi.y;
            const float a = x0 + x2, b = x1 + x3;
            f0[hh] = a + b;
            f2[hh] = a - b;
            fr[hh] = x0 - x2;
            fi[hh] = x3 - x1;
          }
          o0[i] = pack_h2(f0[0], f0[1]);
          o2[i] = pack_h2(f2[0], f2[1]);
          orr[i] = pack_h2(fr[0], fr[1]);
          oi[i] = pack_h2(fi[0], fi[1]);
        }
        // planes: K-major rows of 32 B, 16 B chunk qc at (qc ^ ((r / 4) % 2)) * 16
        uint8_t* pl = smem + OFF_PL + sp * PL_STAGE_BYTES;
        const uint32_t off = r * 32 + ((qc ^ ((r >> 2) & 1)) << 4);
        *reinterpret_cast<uint4*>(pl + 0 * PLANE_BYTES + off) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
        *reinterpret_cast<uint4*>(pl + 1 * PLANE_BYTES + off) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        *reinterpret_cast<uint4*>(pl + 2 * PLANE_BYTES + off) =
            make_uint4(orr[0], orr[1], orr[2], orr[3]);
        *reinterpret_cast<uint4*>(pl + 3 * PLANE_BYTES + off) = make_uint4(oi[0], oi[1], oi[2], oi[3]);
        // make the generic-proxy stores visible to the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pl_full[sp]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

bool fwd_tc_supported(int T, DType dt, int64_t N, int Cin, int Cout) {
  return T == 4 && dt == DType::F16 && N >= 1 && N <= 0x7fffff80LL && Cin % 8 == 0 &&
         Cout % 8 == 0 && Cin >= 8 && Cout >= 8;
}

cudaError_t launch_fwd_tc(int T, const void* X, int64_t N, int Cin, int Cout,
                          const void* Wplanes, const void* bias, void* Y, int* status,
                          int num_sms, cudaStream_t st) {
  if (!fwd_tc_supported(T, DType::F16, N, Cin, Cout)) return cudaErrorNotSupported;
  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;

  CUtensorMap mx, mw;
  {
    cuuint64_t dims[2] = {(cuuint64_t)Cin * kT, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)Cin * kT * 2};
    cuuint32_t box[2] = {64, BM};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(X), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)Cin, (cuuint64_t)Cout, (cuuint64_t)kPlanes};
    cuuint64_t strides[2] = {(cuuint64_t)Cin * 2, (cuuint64_t)Cin * Cout * 2};
    cuuint32_t box[3] = {BK, BD, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(Wplanes), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  TileInfo ti;
  ti.n_dt = (Cout + BD - 1) / BD;
  const int64_t n_rt = (N + BM - 1) / BM;
  if (n_rt * ti.n_dt > 0x7fffffffLL) return cudaErrorInvalidValue;
  ti.num_tiles = (int)(n_rt * ti.n_dt);
  ti.k_stages = (Cin + BK - 1) / BK;

  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(p4_fwd_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = ti.num_tiles < num_sms ? ti.num_tiles : num_sms;
  p4_fwd_tc_kernel<<<grid, kThreads, SMEM_BYTES, st>>>(
      mx, mw, static_cast<const __half*>(bias), static_cast<__half*>(Y), N, Cin, Cout, ti, status);
  return cudaGetLastError();
}

}  // namespace eql
