// tcgen05/TMEM tensor-core forward of the cyclic-group EQ-Linear layer for
// T = 4 (the p4 rotation group) and T = 8, FP16 in, FP32 accumulate, FP16 out,
// for sm_100a.  Also used for dX (the same product with the adjoint weights).
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" items 1-3
// and "Specialisation for p4"): per row n and input channel c the real DFT of
// the group vector x[0..T) (FP32, one rounding to FP16), one real GEMM per real
// frequency and four per complex frequency against the prepared weight planes
// (conjugated spectrum of W), and the inverse DFT plus bias:
//   real k:     Y_k  = X_k A_k^T
//   complex k:  Y_kr = Xr_k Br_k^T - Xi_k Bi_k^T,  Y_ki = Xr_k Bi_k^T + Xi_k Br_k^T
//   y[s] = (Y_0 + (-1)^s Y_{T/2}) / T + (2/T) sum_k (Y_kr cos(2 pi k s/T) - Y_ki sin(2 pi k s/T))
// For T = 4 the transforms are adds only (X0 = x0+x1+x2+x3, X2 = x0-x1+x2-x3,
// Xr = x0-x2, Xi = x3-x1); for T = 8 a radix-2 split leaves one non-dyadic
// twiddle, sqrt(2)/2.  Both operands' planes hold the DFT times 1/T (exact), so
// an FP16 plane never exceeds the largest input magnitude (no overflow for any
// finite FP16 input); the epilogue multiplies the accumulators by T (real
// frequencies) and 2T (complex), which gives the inverse's 1/T and 2/T terms.
//
// Template parameters: ACT = output activation (0 none, 1 GELU, fused into the
// epilogue); IO (T = 4) = spatial X and Y, or Y written as the next layer's
// spectral operand planes [4][N][Cout], or X read as such planes (then the TMA
// box lands directly as the operand planes and the transform warps are idle),
// or spatial X and Y with X's spectrum saved: warp 3 stores transformed stages
// (one TMA box of 32 channels x 128 rows x 4 planes each; stage ks by the
// out-channel tile ks % n_dt) before their slots are released.
//
// Design (one persistent CTA per SM; tile = 128 rows x BD out-channels; K stage
// = BK input channels, whose raw X tile is always 128 rows x 256 B = 32 KB):
//   warp 0      TMA producer: the raw X tile of a stage, one 3-D box
//               (64 halves x 2 row chunks x 128 rows, 128B-swizzled), into a
//               ring of Cfg<T>::X_ST slots (4 at T = 4, 3 at T = 8).
//   warp 2      weight producer: one bulk copy per stage of a blob that
//               prepare_weights pre-arranged in the MMA operand layout, into a
//               ring of Cfg<T>::W_ST slots (2 at T = 4, 6 at T = 8).
//   warp 1      TMEM allocator; lane 0 issues the MMAs of each K step:
//               N = BD for each real frequency, N = 2 BD for Xr_k [Br_k|Bi_k],
//               and N = BD for -Xi_k Bi_k (negate-A bit) and Xi_k Br_k.
//   warps 12-19 transform: group DFT in FP32, one rounding to FP16, written as
//               T K-major swizzled operand planes over the raw tile of the same
//               slot (the planes take exactly the raw tile's 32 KB).
//   warps 4-11  epilogue: the tile's biases staged in shared memory while the
//               main loop runs; tcgen05.ld 32x32b (one row per lane), inverse
//               DFT + bias (+ activation), FP16 pack into a per-warp 4 KB
//               staging buffer, one TMA store per 32 rows x 128 bytes of Y (or
//               per 32 rows x 16 channels x 4 planes for spectral output).
// TMEM (T * BD = 512 columns): real frequency 0 at [0, BD), real frequency T/2
// at [BD, 2 BD), complex frequency k at [2 BD k, 2 BD k + 2 BD) as (re | im).
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the CTA
// sets a shared abort flag and the plan's status word, drains what it issued and
// returns, so a stuck pipeline never hangs the GPU.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"
#include "eql_tc_fwd_parts.cuh"

namespace eql {
namespace {

using namespace tc;
using namespace ftc;

template <int T, int ACT, int IO, int G = 0>
__global__ void __launch_bounds__(kThreads, 1)
    eq_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_y,
                     const __grid_constant__ CUtensorMap map_x_half,
                     const __grid_constant__ CUtensorMap map_y_half,
                     const __grid_constant__ CUtensorMap map_p,
                     const __grid_constant__ CUtensorMap map_p_half,
                     const uint8_t* __restrict__ wtiles, const __half* __restrict__ bias,
                     int64_t N, int Cin, int Cout, TileInfo ti, int* status) {
  using S = Shape<T>;
  constexpr int BD = S::BD;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled TMA destinations and operand tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<T>* bars = reinterpret_cast<Bars<T>*>(smem + S::OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::X_ST; ++s) {
      mbar_init(&bars->x_full[s], 1);          // raw tile landed (TMA bytes)
      mbar_init(&bars->x_read[s], kXfWarps);   // every transform warp holds its raw pieces
      mbar_init(&bars->x_ready[s], kXfWarps);  // operand planes written (transform warps)
      // MMAs done with the planes (tcgen05.commit), and with a saved spectrum its
      // store has read them
      mbar_init(&bars->x_empty[s], IO == kIoSaveSpectrum ? 2 : 1);
    }
    for (int s = 0; s < S::W_ST; ++s) {
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
    // ------- producers: warp 0 raw X (TMA, 3-D box), warp 2 weight tiles (bulk copy) -------
    if (lane == 0) {
      const bool is_raw = (warp == 0);
      const int depth = is_raw ? S::X_ST : S::W_ST;
      uint64_t* full = is_raw ? bars->x_full : bars->w_full;
      uint64_t* empty = is_raw ? bars->x_empty : bars->w_empty;
      int issued_phase[S::X_ST > S::W_ST ? S::X_ST : S::W_ST];  // last phase issued per slot
      for (int s = 0; s < depth; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < ti.num_units; u += gridDim.x) {
        const UnitPos up = unit_pos(u, ti);
        const int row0 = (int)up.row0;
        const int dt = up.dt;
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int s = it % depth;
          const uint32_t ph = (it / depth) & 1;
          if (!(ok = wait_bounded(&empty[s], ph ^ 1, abort_flag, status))) break;
          if (!is_raw && blockIdx.x == 0 && (int)it == ti.drop_w) continue;  // injected fault
          if (is_raw) {
            if constexpr ((IO == kIoSpatial || IO == kIoSaveSpectrum) && T == 4) {
              if (up.half >= 0) {
                // a 64-row half unit: the first 64 rows of the raw layout
                mbar_expect_tx(&full[s], X_STAGE_BYTES / 2);
                tma_load_3d(sbase + S::OFF_X + s * X_STAGE_BYTES, &map_x_half, &full[s], 0,
                            2 * ks, row0);
                issued_phase[s] = (int)ph;
                continue;
              }
            }
            mbar_expect_tx(&full[s], X_STAGE_BYTES);
            if constexpr (IO == kIoSpectralIn) {
              // planes [4][N][Cin] of the previous layer: (32 channels, 128 rows, 4 planes)
              // land as the four K-major 64-byte-swizzled operand planes of this stage
              tma_load_3d(sbase + S::OFF_X + s * X_STAGE_BYTES, &map_x, &full[s], S::BK * ks,
                          row0, 0);
            } else {
              // 3-D view of X: (64 halves, 128-byte chunk of the row, row); a stage is
              // chunks 2ks, 2ks+1 of 128 rows
              tma_load_3d(sbase + S::OFF_X + s * X_STAGE_BYTES, &map_x, &full[s], 0, 2 * ks,
                          row0);
            }
          } else {
            // one pre-arranged blob per (out-channel tile, K stage)
            mbar_expect_tx(&full[s], S::W_STAGE_BYTES);
            const size_t blob = (size_t)dt * ti.k_stages + ks;
            bulk_load(sbase + S::OFF_W + s * S::W_STAGE_BYTES, wtiles + blob * S::W_STAGE_BYTES,
                      S::W_STAGE_BYTES, &full[s]);
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
      for (int u = blockIdx.x; ok && u < ti.num_units; u += gridDim.x, ++tcount) {
        // a half unit (T = 4 only) multiplies its 64 rows with M = 64 MMAs
        int mrows = BM;
        if constexpr (T == 4) mrows = unit_pos(u, ti).half >= 0 ? 64 : BM;
        const uint32_t id_n1 = idesc_f16(mrows, BD);
        const uint32_t id_n1_neg = idesc_f16(mrows, BD, true);
        const uint32_t id_n2 = idesc_f16(mrows, 2 * BD);
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int sx = it % S::X_ST, sw = it % S::W_ST;
          uint64_t* xbar = (IO == kIoSpectralIn) ? &bars->x_full[sx] : &bars->x_ready[sx];
          if (!(ok = wait_bounded(xbar, (it / S::X_ST) & 1, abort_flag, status))) break;
          if (!(ok = wait_bounded(&bars->w_full[sw], (it / S::W_ST) & 1, abort_flag, status)))
            break;
          tc_fence_after();
          const uint32_t pl = sbase + S::OFF_X + sx * X_STAGE_BYTES;     // planes
          const uint32_t wr = sbase + S::OFF_W + sw * S::W_STAGE_BYTES;  // weight regions
#pragma unroll
          for (int kk = 0; kk < S::KSTEPS; ++kk) {
            const uint32_t ko = 32u * kk;  // byte offset of this K step inside the rows
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            auto A = [&](int p) { return desc_kmajor<S::ROWB>(pl + p * S::PLANE_BYTES + ko); };
            auto B = [&](int p) { return desc_kmajor<S::ROWB>(wr + p * S::WREG_BYTES + ko); };
            if constexpr (G == 1) {
              // D4: four characters (N = BD each), then the 2 x 2 block
              // Y[i][k] = sum_j X[i][j] W[k][j]: per (i, j) one N = 2 BD MMA into
              // [Y[i][0] | Y[i][1]] with weight regions 4+2j (k = 0), 5+2j (k = 1)
#pragma unroll
              for (int p = 0; p < 4; ++p) umma(tmem + p * BD, A(p), B(p), id_n1, acc);
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                umma(tmem + 4 * BD + 2 * BD * i, A(4 + 2 * i), B(4), id_n2, acc);
                umma(tmem + 4 * BD + 2 * BD * i, A(5 + 2 * i), B(6), id_n2, 1u);
              }
              continue;
            }
            // real frequencies 0 and T/2
            umma(tmem + 0, A(0), B(0), id_n1, acc);
            umma(tmem + BD, A(1), B(1), id_n1, acc);
            // complex frequencies: [Y_kr|Y_ki] += Xr_k [Br_k|Bi_k]^T ;
            // Y_kr += (-Xi_k) Bi_k^T ; Y_ki += Xi_k Br_k^T
#pragma unroll
            for (int k = 1; k <= S::NC; ++k) {
              const uint32_t col = 2 * BD * k;
              umma(tmem + col, A(2 * k), B(2 * k), id_n2, acc);
              umma(tmem + col, A(2 * k + 1), B(2 * k + 1), id_n1_neg, 1u);
              umma(tmem + col + BD, A(2 * k + 1), B(2 * k), id_n1, 1u);
            }
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
    // Warp w reads TMEM lane quarter q = w % 4 (rows 32q..32q+31 of the tile) and
    // out-channel half ch.  The half goes out in slices of 64/T out-channels: a
    // slice row is 128 contiguous bytes of Y, staged in the warp's 4 KB buffer
    // (128-byte swizzle) and written by one TMA store, so TMEM is free for the
    // next tile as soon as its last slice is read, while the stores drain.
    const int q = warp & 3;
    const int ch = (warp - kEpiWarp0) >> 2;
    uint8_t* stg = smem + S::OFF_STG + (warp - kEpiWarp0) * kStgBytes;
    __half* bsm = reinterpret_cast<__half*>(smem + S::OFF_BIAS + (warp - kEpiWarp0) * 128);
    uint32_t tcount = 0;
    for (int u = blockIdx.x; u < ti.num_units; u += gridDim.x, ++tcount) {
      const UnitPos up = unit_pos(u, ti);
      // M = 128: TMEM lane 32q + l holds row 32q + l; M = 64 (half unit, T = 4 only):
      // lanes 32q .. 32q + 15 hold rows 16q .. 16q + 15
      const bool half = T == 4 && up.half >= 0;
      const int64_t row0 = up.row0 + (half ? 16 * q : 32 * q);
      const int dbase = up.dt * BD + (BD / 2) * ch;
      // stage this warp's BD/2 biases while the mainloop runs (lane l: channels 2l, 2l+1)
      if (2 * lane < BD / 2) {
        const int d = dbase + 2 * lane;
        uint32_t v = 0u;
        if (bias && d < Cout) v = *reinterpret_cast<const uint32_t*>(bias + d);  // Cout even
        reinterpret_cast<uint32_t*>(bsm)[lane] = v;
      }
      __syncwarp();
      if (!warp_wait(&bars->acc_full, tcount & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
      epi_slices<T, BD, ACT, IO, StoreOf<T, IO>, G>(
          lane_addr, ch, lane, stg, bsm, dbase, Cout,
          StoreOf<T, IO>{half ? &map_y_half : &map_y, row0, N});
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else if (IO == kIoSaveSpectrum && warp == 3) {
    // ---------------- spectrum store ----------------
    // Every out-channel tile of a row tile transforms the same X stages; stage ks
    // is stored by tile ks % n_dt, so each tile stores an equal share.  A stored
    // slot is released once the store has read it, checked one stage later
    // (wait_group.read 1) so the store overlaps the next stage.
    if (lane == 0) {
      uint32_t it = 0;
      int pending = -1;  // slot whose store may still be reading it
      bool ok = true;
      for (int u = blockIdx.x; ok && u < ti.num_units; u += gridDim.x) {
        const UnitPos up = unit_pos(u, ti);
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int sx = it % S::X_ST;
          if (!(ok = wait_bounded(&bars->x_ready[sx], (it / S::X_ST) & 1, abort_flag, status)))
            break;
          if (ks % ti.n_dt == up.dt) {
            // the transform warps fenced their plane stores to the async proxy before
            // arriving on x_ready; rows past N and channels past Cin are clipped
            const uint32_t src = sbase + S::OFF_X + sx * X_STAGE_BYTES;
            if (T == 4 && up.half >= 0) {
              // a 64-row half unit fills rows 0..63 of each plane: one box per plane
              for (int p = 0; p < 4; ++p)
                tma_store_3d(&map_p_half, src + p * S::PLANE_BYTES, S::BK * ks, (int)up.row0,
                             p);
            } else {
              tma_store_3d(&map_p, src, S::BK * ks, (int)up.row0, 0);
            }
            bulk_commit();
            if (pending >= 0) {
              bulk_wait_read_1();
              mbar_arrive(&bars->x_empty[pending]);
            }
            pending = sx;
          } else {
            if (pending >= 0) {
              bulk_wait_read_all();
              mbar_arrive(&bars->x_empty[pending]);
              pending = -1;
            }
            mbar_arrive(&bars->x_empty[sx]);
          }
        }
      }
      bulk_wait_all();
      if (pending >= 0) mbar_arrive(&bars->x_empty[pending]);
    }
    __syncwarp();
  } else if (warp >= kXfWarp0 && IO != kIoSpectralIn) {
    // ---------------- transform: group DFT into the operand planes ----------------
    const int xt = threadIdx.x - kXfWarp0 * 32;  // 0..255
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < ti.num_units; u += gridDim.x) {
      // a half unit (T = 4 only) has rows 0..63: threads 128..255 (whole warps) idle
      bool idle = false;
      if constexpr (T == 4) idle = unit_pos(u, ti).half >= 0 && xt >= 128;
      for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
        const int sx = it % S::X_ST;
        if (!(ok = warp_wait(&bars->x_full[sx], (it / S::X_ST) & 1, abort_flag, status))) break;
        uint8_t* slot = smem + S::OFF_X + sx * X_STAGE_BYTES;
        uint4 v[8];
        if (!idle) xf_read<T>(slot, xt, v);
        // every raw piece of the slot is in registers before any plane overwrites it
        // (an mbarrier rather than a named barrier, so the wait stays bounded)
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->x_read[sx]);
        if (!(ok = warp_wait(&bars->x_read[sx], (it / S::X_ST) & 1, abort_flag, status))) break;
        if (!idle) xf_write<T, G>(slot, xt, v);
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


// Re-arrange prepared planes [P][Cout][Cin] into the kernel's per-stage weight
// image: blob (dt, ks) = regions 0..T-1 (prepared planes 0..T-1: real frequency
// 0, real frequency T/2, then Re and Im of each complex frequency), each BD rows
// x BK channels in the K-major swizzled layout the MMAs read; rows and channels
// past the matrix are zero.  One thread per 16-byte piece.  The values are the
// prepared planes unchanged (the DFT times 1/T); the epilogue applies the
// inverse transform's factors.
template <int T>
__global__ void tile_weights_kernel(const __half* __restrict__ planes, int Cin, int Cout,
                                    int n_ks, int64_t n_chunks, uint4* __restrict__ tiles) {
  using S = Shape<T>;
  constexpr int kPieces = S::ROWB / 16;  // 16-byte pieces per row
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_chunks) return;
  const int piece = (int)(idx % kPieces);
  const int r = (int)((idx / kPieces) % S::BD);
  const int region = (int)((idx / kPieces) / S::BD % S::NPL);
  const int64_t blob = (idx / kPieces) / S::BD / S::NPL;
  const int dt = (int)(blob / n_ks), ks = (int)(blob % n_ks);
  const int d = dt * S::BD + r, c0 = ks * S::BK + piece * 8;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (d < Cout && c0 < Cin)  // Cin % 16 == 0: the 8 channels are all in range
    v = *reinterpret_cast<const uint4*>(planes + ((int64_t)region * Cout + d) * Cin + c0);
  // swizzle: piece ^= (byte offset of the row >> 7) within the swizzle span
  const int swz = ((r * S::ROWB) >> 7) & (kPieces - 1);
  const int64_t dst_byte = blob * S::W_STAGE_BYTES + (int64_t)region * S::WREG_BYTES +
                           r * S::ROWB + ((piece ^ swz) << 4);
  tiles[dst_byte >> 4] = v;
}

template <typename F>
cudaError_t dispatch_tc(int T, F&& f) {
  if (T == 4) return f(std::integral_constant<int, 4>{});
  if (T == 8) return f(std::integral_constant<int, 8>{});
  return cudaErrorNotSupported;
}

}  // namespace

bool fwd_tc_supported(int T, DType dt, int64_t N, int Cin, int Cout) {
  return (T == 4 || T == 8) && dt == DType::F16 && N >= 1 && N <= 0x7fffff80LL &&
         Cin % 16 == 0 && Cout % 16 == 0 && Cin >= 16 && Cout >= 16;
}

bool tc_tiles_wanted(int T, DType dt, int C, int D) {
  return (T == 4 || T == 8) && dt == DType::F16 && C % 16 == 0 && D % 16 == 0 && C >= 16 &&
         D >= 16;
}

size_t tc_tile_bytes(int T, int Cin, int Cout) {
  size_t bytes = 0;
  dispatch_tc(T, [&](auto tcst) {
    using S = Shape<decltype(tcst)::value>;
    const size_t n_dt = (size_t)(Cout + S::BD - 1) / S::BD, n_ks = (size_t)(Cin + S::BK - 1) / S::BK;
    bytes = n_dt * n_ks * S::W_STAGE_BYTES;
    return cudaSuccess;
  });
  return bytes;
}

cudaError_t launch_tile_weights(int T, const void* planes, int Cin, int Cout, void* tiles,
                                cudaStream_t st, int group) {
  if (group != 0 && T != 8) return cudaErrorNotSupported;
  return dispatch_tc(T, [&](auto tcst) {
    constexpr int TT = decltype(tcst)::value;
    using S = Shape<TT>;
    const int n_ks = (Cin + S::BK - 1) / S::BK;
    const int64_t n_chunks = (int64_t)tc_tile_bytes(TT, Cin, Cout) / 16;
    const unsigned blocks = (unsigned)((n_chunks + 255) / 256);
    tile_weights_kernel<TT><<<blocks, 256, 0, st>>>(static_cast<const __half*>(planes), Cin, Cout,
                                                    n_ks, n_chunks, static_cast<uint4*>(tiles));
    return cudaGetLastError();
  });
}

namespace {

// Spectral planes [4][N][channels] (FP16), viewed as (channel, row, plane).
bool encode_planes_map(CUtensorMap* m, void* base, int channels, int64_t N, uint32_t box_ch,
                       uint32_t box_rows, CUtensorMapSwizzle swz, uint32_t box_planes = 4) {
  auto encode = encode_fn();
  cuuint64_t dims[3] = {(cuuint64_t)channels, (cuuint64_t)N, 4};
  cuuint64_t strides[2] = {(cuuint64_t)channels * 2, (cuuint64_t)N * channels * 2};
  cuuint32_t box[3] = {box_ch, box_rows, box_planes};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int TT, int ACT, int IO, int G = 0>
cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(eq_fwd_tc_kernel<TT, ACT, IO, G>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, Shape<TT>::SMEM_BYTES);
}

// D4 weight spectrum, in the tile regions' order: W^(rho) = sum_u W(u) rho(u)
// for the characters (+,+), (+,-), (-,+), (-,-) and the 2 x 2 entries 00, 10,
// 01, 11 (region 4 + 2j + k holds entry [k][j]), times 1/8 like every stored
// plane (exact); FP32, one rounding.
// W [D][C][8] -> planes [8][D][C].  One thread per (d, c).
__global__ void prepare_d4_kernel(const __half* __restrict__ W, int C, int D,
                                  __half* __restrict__ planes) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t plane = (int64_t)C * D;
  if (idx >= plane) return;
  float x[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) x[u] = __half2float(W[idx * 8 + u]);
  const float e0 = x[0] + x[2], o0 = x[1] + x[3], e1 = x[4] + x[6], o1 = x[5] + x[7];
  const float d0 = x[0] - x[2], d1 = x[1] - x[3], d4 = x[4] - x[6], d5 = x[5] - x[7];
  const float v[8] = {(e0 + o0) + (e1 + o1), (e0 + o0) - (e1 + o1), (e0 - o0) + (e1 - o1),
                      (e0 - o0) - (e1 - o1),
                      d0 + d4,   // [0][0]
                      d1 + d5,   // [1][0]
                      d5 - d1,   // [0][1]
                      d0 - d4};  // [1][1]
#pragma unroll
  for (int r = 0; r < 8; ++r) planes[r * plane + idx] = __float2half_rn(v[r] * 0.125f);
}

}  // namespace

cudaError_t launch_prepare_d4(const void* W, int C, int D, void* planes, cudaStream_t st) {
  const int64_t total = (int64_t)C * D;
  prepare_d4_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
      static_cast<const __half*>(W), C, D, static_cast<__half*>(planes));
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc(int T, const void* X, int64_t N, int Cin, int Cout,
                          const void* Wtiles, const void* bias, void* Y, int* status,
                          int num_sms, int drop_w_stage, int act, int io, cudaStream_t st,
                          int group, void* spectrum) {
  if (!fwd_tc_supported(T, DType::F16, N, Cin, Cout)) return cudaErrorNotSupported;
  if (!Wtiles) return cudaErrorNotSupported;
  if (io != kIoSpatial && T != 4) return cudaErrorNotSupported;
  if ((io == kIoSaveSpectrum) != (spectrum != nullptr)) return cudaErrorInvalidValue;
  if (group != 0 && (T != 8 || io != kIoSpatial)) return cudaErrorNotSupported;
  if (act != 0 && act != 1) return cudaErrorInvalidValue;

  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  return dispatch_tc(T, [&](auto tcst) {
    constexpr int TT = decltype(tcst)::value;
    using S = Shape<TT>;
    cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap mx, mx_half, my_half;
    if (io == kIoSpectralIn) {
      // planes of the previous layer: box = 32 channels (64 B) x 128 rows x 4 planes
      if (!encode_planes_map(&mx, const_cast<void*>(X), Cin, N, S::BK, BM,
                             CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    } else {
      // X row = Cin*T/64 chunks of 64 halves (128 B); box = 2 chunks x 128 rows
      cuuint64_t dims[3] = {64, (cuuint64_t)Cin * TT / 64, (cuuint64_t)N};
      cuuint64_t strides[2] = {128, (cuuint64_t)Cin * TT * 2};
      cuuint32_t box[3] = {64, 2, BM};
      if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(X), dims, strides,
                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
      // half units: 64 rows
      cuuint32_t hbox[3] = {64, 2, 64};
      if (encode(&mx_half, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(X), dims,
                 strides, hbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    CUtensorMap my;
    if (io == kIoSpectralOut) {
      // planes for the next layer: store box = 16 channels (32 B) x 32 rows x 4 planes
      if (!encode_planes_map(&my, Y, Cout, N, 16, 32, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    } else {
      // Y row = Cout*T/64 chunks of 128 B; store box = 1 chunk x 32 rows
      cuuint64_t ydims[3] = {64, (cuuint64_t)Cout * TT / 64, (cuuint64_t)N};
      cuuint64_t ystrides[2] = {128, (cuuint64_t)Cout * TT * 2};
      cuuint32_t ybox[3] = {64, 1, 32};
      if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, Y, ydims, ystrides, ybox, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
      // half units: an epilogue warp stores 16 rows
      cuuint32_t yhbox[3] = {64, 1, 16};
      if (encode(&my_half, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, Y, ydims, ystrides, yhbox, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    CUtensorMap mp = mx, mp_half = mx;
    if (io == kIoSaveSpectrum) {
      // the input's spectrum: store box = 32 channels (64 B) x 128 rows x 4 planes,
      // for half units 32 channels x 64 rows x 1 plane
      if (!encode_planes_map(&mp, spectrum, Cin, N, S::BK, BM, CU_TENSOR_MAP_SWIZZLE_64B) ||
          !encode_planes_map(&mp_half, spectrum, Cin, N, S::BK, 64, CU_TENSOR_MAP_SWIZZLE_64B,
                             1))
        return cudaErrorInvalidValue;
    }
    const bool halves_ok = io == kIoSpatial || io == kIoSaveSpectrum;
    if (!halves_ok) {  // no half units with spectral input or output
      mx_half = mx;
      my_half = my;
    }
    TileInfo ti;
    ti.n_dt = (Cout + S::BD - 1) / S::BD;
    const int64_t n_rt = (N + BM - 1) / BM;
    if (n_rt * ti.n_dt > 0x7fffffffLL) return cudaErrorInvalidValue;
    ti.num_tiles = (int)(n_rt * ti.n_dt);
    ti.k_stages = (Cin + S::BK - 1) / S::BK;
    ti.drop_w = drop_w_stage;
    // The last partial wave (rem tiles) runs as 2 * rem half units when that still
    // fits in one wave: a half unit moves about 0.6 of a tile's shared-memory
    // traffic (its MMAs cost as much as a whole tile's), so the wave ends sooner.
    ti.full = ti.num_tiles;
    ti.num_units = ti.num_tiles;
    if (halves_ok && TT == 4) {  // T = 8 tiles keep their registers for the transform
      const int rem = ti.num_tiles >= num_sms ? ti.num_tiles % num_sms : ti.num_tiles;
      if (rem > 0 && 2 * rem <= num_sms) {
        ti.full = ti.num_tiles - rem;
        ti.num_units = ti.full + 2 * rem;
      }
    }
    static bool attr_set = false;
    if (!attr_set) {
      cudaError_t e = set_smem_attr<TT, 0, kIoSpatial>();
      if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSpatial>();
      if constexpr (TT == 4) {
        if (e == cudaSuccess) e = set_smem_attr<TT, 0, kIoSpectralOut>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSpectralOut>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 0, kIoSpectralIn>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSpectralIn>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 0, kIoSaveSpectrum>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSaveSpectrum>();
      } else {
        if (e == cudaSuccess) e = set_smem_attr<TT, 0, kIoSpatial, 1>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSpatial, 1>();
      }
      if (e != cudaSuccess) return e;
      attr_set = true;
    }
    const int grid = ti.num_units < num_sms ? ti.num_units : num_sms;
    auto kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSpatial> : eq_fwd_tc_kernel<TT, 0, kIoSpatial>;
    if constexpr (TT == 4) {
      if (io == kIoSpectralOut)
        kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSpectralOut>
                          : eq_fwd_tc_kernel<TT, 0, kIoSpectralOut>;
      else if (io == kIoSpectralIn)
        kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSpectralIn>
                          : eq_fwd_tc_kernel<TT, 0, kIoSpectralIn>;
      else if (io == kIoSaveSpectrum)
        kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSaveSpectrum>
                          : eq_fwd_tc_kernel<TT, 0, kIoSaveSpectrum>;
    } else {
      if (group == 1)
        kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSpatial, 1>
                          : eq_fwd_tc_kernel<TT, 0, kIoSpatial, 1>;
    }
    kernel<<<grid, kThreads, S::SMEM_BYTES, st>>>(
        mx, my, mx_half, my_half, mp, mp_half, static_cast<const uint8_t*>(Wtiles),
        static_cast<const __half*>(bias), N, Cin, Cout, ti, status);
    return cudaGetLastError();
  });
}

}  // namespace eql
