// tcgen05/TMEM tensor-core forward of the p4 (T = 4) EQ-Linear layer, FP16 in,
// FP32 accumulate, FP16 out, for sm_100a.
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" and
// "Specialisation for p4"): per row n and input channel c the group DFT
//   X0 = x0+x1+x2+x3,  X2 = x0-x1+x2-x3,  Xr = x0-x2,  Xi = x3-x1
// (adds only), six real GEMMs against the prepared weight planes
//   Y0 = X0 A0^T,  Y2 = X2 A2^T,
//   Y1r = Xr Br^T - Xi Bi^T,  Y1i = Xr Bi^T + Xi Br^T
// and the inverse DFT with the dyadic factors 1/4 and 1/2, plus bias:
//   y0 = (Y0+Y2)/4 + Y1r/2,  y1 = (Y0-Y2)/4 - Y1i/2,
//   y2 = (Y0+Y2)/4 - Y1r/2,  y3 = (Y0-Y2)/4 + Y1i/2.
//
// Design (one persistent CTA per SM, tile = 128 rows x 128 out-channels, K
// stages of 16 input channels = one MMA K step):
//   warp 0      TMA producer: the raw X tile of a stage (128 rows x 16 channels
//               x 4, one 128B-swizzled box) into the X ring.
//   warp 2      weight producer: one bulk copy per stage of a 16 KB blob that
//               prepare_weights pre-arranged in the operand layout (A0, A2, Br, Bi).
//   warp 1      TMEM allocator; lane 0 issues the five tcgen05.mma of a stage:
//               N = 128 for Y0 and Y2, N = 256 for Xr [Br|Bi], and two N = 128
//               for -Xi Bi (negate-A bit) and Xi Br.
//   warps 12-19 transform: group DFT in FP32, one rounding to FP16, written as
//               four K-major 32B-swizzled operand planes over the raw tile of the
//               same slot (the planes take exactly the raw tile's 16 KB).
//   warps 4-11  epilogue: tcgen05.ld of the four accumulators, inverse DFT, bias,
//               FP16 pack, 16-byte global stores.
// Accumulators in TMEM: Y0 at columns [0,128), Y2 [128,256), Y1r [256,384),
// Y1i [384,512).  Every mbarrier wait is bounded (about 2 s of %globaltimer); on
// expiry the CTA sets a shared abort flag and the plan's status word, drains
// what it issued and returns, so a stuck pipeline never hangs the GPU.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "eql_kernels.h"

namespace eql {
namespace {

constexpr int kT = 4;
constexpr int BM = 128;          // rows per tile = MMA M
constexpr int BD = 128;          // out-channels per tile
constexpr int BK = 32;           // in-channels per pipeline stage = two MMA K steps
constexpr int X_ST = 4;          // X ring: raw tile in, transformed operand planes out (in place)
constexpr int W_ST = 3;          // weight-tile ring (L2-resident source)
constexpr int kPlanes = 4;       // A0, A2, Br, Bi
constexpr int kThreads = 640;
constexpr int kEpiWarp0 = 4;     // warps 4..11: two per TMEM lane quarter
constexpr int kEpiWarps = 8;
constexpr int kXfWarp0 = 12;     // warps 12..19
constexpr int kXfWarps = 8;
constexpr uint32_t kTmemCols = 4 * BD;  // 512

// One 32 KB TMA op per stage for X and one 32 KB bulk op for the weights: the
// per-SM load rate grows with the bytes each operation carries.
constexpr uint32_t X_STAGE_BYTES = BM * BK * kT * 2;      // 128 rows x 32 channels x 4 x 2 B
constexpr uint32_t PLANE_BYTES = BM * BK * 2;             // 128 rows x 64 B
static_assert(4 * PLANE_BYTES == X_STAGE_BYTES, "the four planes replace the raw tile in place");
constexpr uint32_t WREG_BYTES = BD * BK * 2;              // BD rows x 64 B
constexpr uint32_t W_STAGE_BYTES = kPlanes * WREG_BYTES;
constexpr uint32_t OFF_X = 0;
constexpr uint32_t OFF_W = OFF_X + X_ST * X_STAGE_BYTES;
constexpr uint32_t OFF_BAR = OFF_W + W_ST * W_STAGE_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;     // barriers + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

constexpr unsigned long long kTimeoutNs = 2000000000ull;

// status word codes
constexpr int kErrTimeout = 1;

struct Bars {
  uint64_t x_full[X_ST], x_read[X_ST], x_ready[X_ST], x_empty[X_ST];
  uint64_t w_full[W_ST], w_empty[W_ST];
  uint64_t acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");

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
// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `ns` nanoseconds pass, instead of spinning on shared
// memory (which would steal issue slots from the producer and MMA threads).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* b, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Bounded wait: false if the CTA aborted or the wait timed out (then aborts it).
__device__ __noinline__ bool wait_bounded(uint64_t* b, uint32_t parity, Bars* bars, int* status) {
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = gtimer();
  while (true) {
    if (mbar_try_wait_sleep(b, parity, 200000u)) return true;
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
  while (!mbar_try_wait_sleep(b, parity, 200000u)) {
    if (gtimer() - t0 > kTimeoutNs) return;
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Plain bulk copy global -> shared of `bytes` (multiple of 16, both 16 B aligned).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// K-major, 64-byte-swizzled operand tile: rows of 64 B (32 fp16 of K), 8-row
// groups 512 B apart (SBO), descriptor version 1 (sm_100), layout type 4
// (SWIZZLE_64B: 16-byte chunk index ^= (row / 2) % 4).  The second MMA K step of
// a stage starts 32 B into the rows.
__device__ __forceinline__ uint64_t desc_kmajor_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;              // leading byte offset (unused when swizzled)
  d |= (uint64_t)(512u >> 4) << 32;     // stride byte offset: 8 rows x 64 B
  d |= (uint64_t)1u << 46;              // descriptor version for sm_100
  d |= (uint64_t)4u << 61;              // SWIZZLE_64B
  return d;
}
// Instruction descriptor, kind::f16: A = B = F16, D = F32, both K-major;
// bit 13 negates A.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool negate_a = false) {
  return (1u << 4) | (negate_a ? (1u << 13) : 0u) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
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
// The .x2 form repeats the pattern for the next 8 columns in regs 4..7.
#define EQL_TMEM_LD_16x256_X2(taddr, r)                                                    \
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"    \
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),    \
                 "=r"(r[6]), "=r"(r[7])                                                    \
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
  int drop_w;     // fault injection for tests: CTA 0 never issues weight stage drop_w (-1: off)
};

__global__ void __launch_bounds__(kThreads, 1)
    p4_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                     const uint8_t* __restrict__ wtiles, const __half* __restrict__ bias,
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
    for (int s = 0; s < X_ST; ++s) {
      mbar_init(&bars->x_full[s], 1);          // raw tile landed (TMA bytes)
      mbar_init(&bars->x_read[s], kXfWarps);   // every transform warp holds its raw chunks
      mbar_init(&bars->x_ready[s], kXfWarps);  // operand planes written (transform warps)
      mbar_init(&bars->x_empty[s], 1);         // MMAs done with the planes (tcgen05.commit)
    }
    for (int s = 0; s < W_ST; ++s) {
      mbar_init(&bars->w_full[s], 1);
      mbar_init(&bars->w_empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kEpiWarps * 32);
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
    // ------- producers: warp 0 raw X (TMA, 2D box), warp 2 weight tiles (bulk copy) -------
    if (lane == 0) {
      const bool is_raw = (warp == 0);
      const int depth = is_raw ? X_ST : W_ST;
      uint64_t* full = is_raw ? bars->x_full : bars->w_full;
      uint64_t* empty = is_raw ? bars->x_empty : bars->w_empty;
      int issued_phase[X_ST > W_ST ? X_ST : W_ST];  // last phase issued per slot
      for (int s = 0; s < depth; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x) {
        const int row0 = (tile / ti.n_dt) * BM;
        const int d0 = (tile % ti.n_dt) * BD;
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int s = it % depth;
          const uint32_t ph = (it / depth) & 1;
          if (!(ok = wait_bounded(&empty[s], ph ^ 1, bars, status))) break;
          if (!is_raw && blockIdx.x == 0 && (int)it == ti.drop_w) continue;  // injected fault
          if (is_raw) {
            mbar_expect_tx(&full[s], X_STAGE_BYTES);
            // 3-D view of X: (64 halves, 128-byte chunk of the row, row); a stage is
            // chunks 2ks, 2ks+1 of 128 rows
            tma_load_3d(sbase + OFF_X + s * X_STAGE_BYTES, &map_x, &full[s], 0, 2 * ks, row0);
          } else {
            // one pre-arranged blob per (out-channel tile, K stage): regions
            // A0, A2, Br, Bi in the operand layout the MMAs read
            mbar_expect_tx(&full[s], W_STAGE_BYTES);
            const size_t blob = (size_t)(d0 / BD) * ti.k_stages + ks;
            bulk_load(sbase + OFF_W + s * W_STAGE_BYTES, wtiles + blob * W_STAGE_BYTES,
                      W_STAGE_BYTES, &full[s]);
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
      const uint32_t id_n1_neg = idesc_f16(BM, BD, true);
      const uint32_t id_n2 = idesc_f16(BM, 2 * BD);
      for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x, ++tcount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, bars, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int sx = it % X_ST, sw = it % W_ST;
          if (!(ok = wait_bounded(&bars->x_ready[sx], (it / X_ST) & 1, bars, status))) break;
          if (!(ok = wait_bounded(&bars->w_full[sw], (it / W_ST) & 1, bars, status))) break;
          tc_fence_after();
          const uint32_t pl = sbase + OFF_X + sx * X_STAGE_BYTES;   // planes X0, X2, Xr, Xi
          const uint32_t wr = sbase + OFF_W + sw * W_STAGE_BYTES;   // regions A0, A2, Br, Bi
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t ko = 32u * kk;  // byte offset of this K step inside the 64 B rows
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            // Y0 += X0 A0^T ; Y2 += X2 A2^T ; [Y1r|Y1i] += Xr [Br|Bi]^T ;
            // Y1r += (-Xi) Bi^T ; Y1i += Xi Br^T
            umma(tmem + 0, desc_kmajor_sw64(pl + 0 * PLANE_BYTES + ko),
                 desc_kmajor_sw64(wr + 0 * WREG_BYTES + ko), id_n1, acc);
            umma(tmem + BD, desc_kmajor_sw64(pl + 1 * PLANE_BYTES + ko),
                 desc_kmajor_sw64(wr + 1 * WREG_BYTES + ko), id_n1, acc);
            umma(tmem + 2 * BD, desc_kmajor_sw64(pl + 2 * PLANE_BYTES + ko),
                 desc_kmajor_sw64(wr + 2 * WREG_BYTES + ko), id_n2, acc);
            umma(tmem + 2 * BD, desc_kmajor_sw64(pl + 3 * PLANE_BYTES + ko),
                 desc_kmajor_sw64(wr + 3 * WREG_BYTES + ko), id_n1_neg, 1u);
            umma(tmem + 3 * BD, desc_kmajor_sw64(pl + 3 * PLANE_BYTES + ko),
                 desc_kmajor_sw64(wr + 2 * WREG_BYTES + ko), id_n1, 1u);
          }
          umma_commit(&bars->x_empty[sx]);
          umma_commit(&bars->w_empty[sw]);
        }
        if (ok) umma_commit(&bars->acc_full);
      }
      // all MMAs this thread issued must be complete before TMEM is freed
      umma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
    // ---------------- epilogue ----------------
    // Warp w reads TMEM lane quarter q = w % 4 (rows 32q..32q+31) and column half
    // ch (out-channels 64ch..64ch+63 of the tile).  16x256b loads give lane t
    // rows (t/4, t/4 + 8) of a 16-lane group and out-channel pair 2*(t%4) of
    // each 8-channel group, so each 16-byte store of a warp covers 8 rows x 64
    // contiguous bytes.
    const int q = warp & 3;
    const int ch = (warp - kEpiWarp0) >> 2;
    uint32_t tcount = 0;
    const int64_t ldy = (int64_t)Cout * kT;
    const int tr = lane >> 2, tc = 2 * (lane & 3);
    for (int tile = blockIdx.x; tile < ti.num_tiles; tile += gridDim.x, ++tcount) {
      const int64_t rbase = (int64_t)(tile / ti.n_dt) * BM + 32 * q;
      const int dbase = (tile % ti.n_dt) * BD + 64 * ch;
      // bias of this lane's 16 out-channels, loaded while the mainloop runs
      float2 bv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int d = dbase + 8 * j + tc;
        bv[j] = (bias && d < Cout) ? __half22float2(*reinterpret_cast<const __half2*>(bias + d))
                                   : make_float2(0.f, 0.f);
      }
      if (!warp_wait(&bars->acc_full, tcount & 1, bars, status)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {  // 16-lane groups of the quarter
        const uint32_t laddr = tmem + ((uint32_t)(32 * q + 16 * h) << 16) + 64 * ch;
        const int64_t row_a = rbase + 16 * h + tr, row_b = row_a + 8;
#pragma unroll
        for (int bt = 0; bt < 4; ++bt) {  // 16-column batches
          uint32_t a0[8], a2[8], ar[8], ai[8];
          EQL_TMEM_LD_16x256_X2(laddr + 16 * bt, a0);
          EQL_TMEM_LD_16x256_X2(laddr + BD + 16 * bt, a2);
          EQL_TMEM_LD_16x256_X2(laddr + 2 * BD + 16 * bt, ar);
          EQL_TMEM_LD_16x256_X2(laddr + 3 * BD + 16 * bt, ai);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int g = 0; g < 2; ++g) {  // 8-column group inside the batch
            const int j = 2 * bt + g;
            const int d = dbase + 8 * j + tc;
            if (d >= Cout) continue;  // warp-uniform: Cout is a multiple of 8
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
              const int64_t row = rr ? row_b : row_a;
              if (row >= N) continue;
              uint32_t packed[4];
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {  // out-channel d + hh
                const int k = 4 * g + 2 * rr + hh;
                const float y0 = __uint_as_float(a0[k]), y2 = __uint_as_float(a2[k]);
                const float yr = __uint_as_float(ar[k]), yi = __uint_as_float(ai[k]);
                const float bb = hh ? bv[j].y : bv[j].x;
                const float e = (y0 + y2) * 0.25f, o = (y0 - y2) * 0.25f;
                const float r = yr * 0.5f, m = yi * 0.5f;
                packed[2 * hh + 0] = pack_h2(e + r + bb, o - m + bb);
                packed[2 * hh + 1] = pack_h2(e - r + bb, o + m + bb);
              }
              *reinterpret_cast<uint4*>(Y + row * ldy + (int64_t)d * kT) =
                  make_uint4(packed[0], packed[1], packed[2], packed[3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
  } else if (warp >= kXfWarp0) {
    // ---------------- transform: group DFT into the operand planes ----------------
    // The raw stage is [row][128-byte chunk c of 16 channels][128 B], every
    // 128-byte line L = 2r + c swizzled by (L % 8).  One unit = one row x 8
    // channels (half hq of chunk c): four 16-byte raw pieces in, one 16-byte piece
    // out per plane (K-major 64 B rows, piece q = 2c + hq at (q ^ ((r/2) % 4))).
    // An 8-lane phase covers 4 rows x both chunks, so its swizzled reads and
    // writes hit 8 distinct bank groups.  Planes overwrite the raw tile of the
    // same slot once every transform warp holds its raw pieces.
    const int xt = threadIdx.x - kXfWarp0 * 32;  // 0..255
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x) {
      for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
        const int sx = it % X_ST;
        if (!(ok = warp_wait(&bars->x_full[sx], (it / X_ST) & 1, bars, status))) break;
        uint8_t* slot = smem + OFF_X + sx * X_STAGE_BYTES;
        uint4 v[2][4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int unit = xt + 256 * u;
          const int c = unit & 1, r = (unit >> 1) & (BM - 1), hq = unit >> 8;
          const int line = 2 * r + c;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int j = hq * 4 + i;
            v[u][i] = *reinterpret_cast<const uint4*>(slot + line * 128 + ((j ^ (line & 7)) << 4));
          }
        }
        // every raw piece of the slot is in registers before any plane overwrites it
        // (an mbarrier rather than a named barrier, so the wait stays bounded)
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->x_read[sx]);
        if (!(ok = warp_wait(&bars->x_read[sx], (it / X_ST) & 1, bars, status))) break;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int unit = xt + 256 * u;
          const int c = unit & 1, r = (unit >> 1) & (BM - 1), hq = unit >> 8;
          const int q = 2 * c + hq;
          // piece i holds channels 2i (.x = x0,x1  .y = x2,x3) and 2i+1 (.z, .w)
          uint32_t o0[4], o2[4], orr[4], oi[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f0[2], f2[2], fr[2], fi[2];
            const uint32_t w4[4] = {v[u][i].x, v[u][i].y, v[u][i].z, v[u][i].w};
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
          const uint32_t off = r * 64 + ((q ^ ((r >> 1) & 3)) << 4);
          *reinterpret_cast<uint4*>(slot + 0 * PLANE_BYTES + off) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
          *reinterpret_cast<uint4*>(slot + 1 * PLANE_BYTES + off) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
          *reinterpret_cast<uint4*>(slot + 2 * PLANE_BYTES + off) =
              make_uint4(orr[0], orr[1], orr[2], orr[3]);
          *reinterpret_cast<uint4*>(slot + 3 * PLANE_BYTES + off) = make_uint4(oi[0], oi[1], oi[2], oi[3]);
        }
        // make the generic-proxy stores visible to the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->x_ready[sx]);
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
  return T == 4 && dt == DType::F16 && N >= 1 && N <= 0x7fffff80LL && Cin % 16 == 0 &&
         Cout % 16 == 0 && Cin >= 16 && Cout >= 16;
}

bool tc_tiles_wanted(int T, DType dt, int C, int D) {
  return T == 4 && dt == DType::F16 && C % 16 == 0 && D % 16 == 0 && C >= 16 && D >= 16;
}

size_t tc_tile_bytes(int Cin, int Cout) {
  const size_t n_dt = (size_t)(Cout + BD - 1) / BD, n_ks = (size_t)(Cin + BK - 1) / BK;
  return n_dt * n_ks * W_STAGE_BYTES;
}

namespace {
// Re-arrange prepared planes [P][Cout][Cin] into the kernel's per-stage weight
// image: blob (dt, ks) = regions A0, A2, Br, Bi (prepared planes 0..3), each BD
// rows x 32 channels in the K-major 64B-swizzled layout; rows and channels past
// the matrix are zero.  One thread per 16-byte chunk.
__global__ void tile_weights_kernel(const __half* __restrict__ planes, int Cin, int Cout,
                                    int n_ks, int64_t n_chunks, uint4* __restrict__ tiles) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_chunks) return;
  const int chunk = (int)(idx & 3);                   // 8-channel piece of the 64 B row
  const int r = (int)((idx >> 2) % BD);               // row in the region
  const int region = (int)((idx >> 2) / BD % kPlanes);
  const int64_t blob = (idx >> 2) / BD / kPlanes;
  const int dt = (int)(blob / n_ks), ks = (int)(blob % n_ks);
  const int d = dt * BD + r, c0 = ks * BK + chunk * 8;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (d < Cout && c0 < Cin)  // Cin % 8 == 0: the 8 channels are all in range
    v = *reinterpret_cast<const uint4*>(planes + ((int64_t)region * Cout + d) * Cin + c0);
  const int64_t dst_byte = blob * W_STAGE_BYTES + (int64_t)region * WREG_BYTES + r * 64 +
                           ((chunk ^ ((r >> 1) & 3)) << 4);
  tiles[dst_byte >> 4] = v;
}
}  // namespace

cudaError_t launch_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                cudaStream_t st) {
  const int n_ks = (Cin + BK - 1) / BK;
  const int64_t n_chunks = (int64_t)tc_tile_bytes(Cin, Cout) / 16;
  const unsigned blocks = (unsigned)((n_chunks + 255) / 256);
  tile_weights_kernel<<<blocks, 256, 0, st>>>(static_cast<const __half*>(planes), Cin, Cout,
                                               n_ks, n_chunks, static_cast<uint4*>(tiles));
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc(int T, const void* X, int64_t N, int Cin, int Cout,
                          const void* Wtiles, const void* bias, void* Y, int* status,
                          int num_sms, int drop_w_stage, cudaStream_t st) {
  if (!fwd_tc_supported(T, DType::F16, N, Cin, Cout)) return cudaErrorNotSupported;
  if (!Wtiles) return cudaErrorNotSupported;
  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;

  CUtensorMap mx;
  {
    // X row = Cin/16 chunks of 64 halves (128 B); box = 2 chunks x 128 rows
    cuuint64_t dims[3] = {64, (cuuint64_t)Cin / 16, (cuuint64_t)N};
    cuuint64_t strides[2] = {128, (cuuint64_t)Cin * kT * 2};
    cuuint32_t box[3] = {64, 2, BM};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(X), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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
  ti.drop_w = drop_w_stage;

  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(p4_fwd_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int grid = ti.num_tiles < num_sms ? ti.num_tiles : num_sms;
  p4_fwd_tc_kernel<<<grid, kThreads, SMEM_BYTES, st>>>(
      mx, static_cast<const uint8_t*>(Wtiles), static_cast<const __half*>(bias),
      static_cast<__half*>(Y), N, Cin, Cout, ti, status);
  return cudaGetLastError();
}

}  // namespace eql
