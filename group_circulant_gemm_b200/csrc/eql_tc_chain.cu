// Two chained p4 (T = 4) EQ-Linear layers in one persistent tcgen05 launch:
// H = act(L1(X)), Y = L2(H), FP16 in, FP32 accumulate, FP16 out.
//
// What it computes is exactly what two one-layer calls compute (Flash
// EQ-Linear summary, "Algorithmic approach" and "Specialisation for p4"; the
// two layers are the MLP pair of a Flash EQ-ViT block): every tile runs the
// same transform, MMAs and epilogue as eq_fwd_tc_kernel<4>, in the same order,
// so H and Y are bitwise the outputs of the two separate calls.  Only the
// scheduling differs.  Each layer alone leaves SMs idle at its end (ViT-B: 594
// layer-1 tiles, 198 layer-2 tiles on 148 SMs); here both layers' tiles form
// one queue that the CTAs take from dynamically (a global atomic counter), so
// the SMs that finish early keep working.
//
// Queue order: the layer-1 tiles of the first `lag` row tiles, then per row tile
// k the layer-1 tiles of row k followed by the layer-2 tiles of row k - lag, then
// the remaining layer-2 tiles.  The lag (about 0.6 of the row tiles, at least one
// wave) came from simulating the queue with measured tile times: a short lag
// leaves many long layer-2 tiles for the end, a long one starts them late.
//
// A layer-2 tile of row r reads the whole H row tile r, so before loading it
// the X producer waits (bounded) until
// that row's counter shows every layer-1 tile of row r stored: each epilogue
// warp, once its TMA stores of a layer-1 tile are complete, adds 1 (release,
// GPU scope).  Every layer-1 tile of row r sits earlier in the queue than any
// layer-2 tile of row r, so it was taken by a running CTA (the grid is at most
// one CTA per SM, all resident) and completes: the waits cannot form a cycle.
//
// Within a CTA the X producer takes each task from the counter and hands its
// number to the other roles through a 4-deep shared-memory ring (one mbarrier
// pair per slot); the roles are those of eq_fwd_tc_kernel.  The intermediate H
// is spatial [N][C1*4] or, with SPEC, the layer-1 epilogue writes the group DFT
// of act(y) as operand planes [4][N][C1] that layer 2 loads without a transform.
//
// Counters (int32, the caller's workspace): [0] next task, [1] CTAs finished,
// [2 + r] row tile r.  They must be zero when the kernel starts; the last CTA to
// finish sets them back to zero, so a zero-filled workspace stays ready for the
// next call.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"
#include "eql_tc_fwd_parts.cuh"

namespace eql {
namespace {

using namespace tc;
using namespace ftc;

using S = Shape<4>;
constexpr int BD = S::BD;
constexpr int kQ = 4;  // task ring depth
// readers of each task: W producer, MMA issuer, 8 epilogue warps, 8 transform warps
constexpr int kTaskReaders = 2 + kEpiWarps + kXfWarps;

struct ChainInfo {
  int64_t N;
  int C0, C1, C2;    // layer 1: C0 -> C1 channels; layer 2: C1 -> C2
  int n_rt;          // row tiles of 128 rows
  int n_dt1, n_dt2;  // out-channel tiles per layer
  int ks1, ks2;      // K stages per layer
  int lag;           // layer-1 row tiles queued ahead of layer 2
  int total;         // tasks
  int flag_target;   // counter value of a complete layer-1 row tile (8 per tile)
};

struct TaskRing {
  uint64_t full[kQ], empty[kQ];
  int id[kQ];
};

struct Task {
  int layer, r, j;
};

__device__ __forceinline__ Task decode(int q, const ChainInfo& ci) {
  Task t;
  const int a = ci.lag * ci.n_dt1;
  const int per = ci.n_dt1 + ci.n_dt2;
  const int b = (ci.n_rt - ci.lag) * per;
  if (q < a) {
    t.layer = 0; t.r = q / ci.n_dt1; t.j = q % ci.n_dt1;
  } else if (q < a + b) {
    const int qq = q - a, k = ci.lag + qq / per, o = qq % per;
    if (o < ci.n_dt1) {
      t.layer = 0; t.r = k; t.j = o;
    } else {
      t.layer = 1; t.r = k - ci.lag; t.j = o - ci.n_dt1;
    }
  } else {
    const int qq = q - a - b;
    t.layer = 1; t.r = ci.n_rt - ci.lag + qq / ci.n_dt2; t.j = qq % ci.n_dt2;
  }
  return t;
}

// Bounded wait until a layer-1 row tile is complete, then order the TMA loads
// that follow after the acquire.
__device__ __noinline__ bool wait_row(const int* flag, int target, int* abort_flag, int* status) {
  const uint64_t t0 = gtimer();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v >= target) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
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

// Read the next task number from the ring (one thread); -1 ends the sequence.
__device__ __forceinline__ bool ring_take(TaskRing* ring, uint32_t n, int* id, int* abort_flag,
                                          int* status) {
  const int s = n % kQ;
  if (!wait_bounded(&ring->full[s], (n / kQ) & 1, abort_flag, status)) return false;
  *id = *(volatile int*)&ring->id[s];
  mbar_arrive(&ring->empty[s]);
  return true;
}
// Same for a whole warp: every lane gets the number, lane 0 releases the slot.
__device__ __forceinline__ bool ring_take_warp(TaskRing* ring, uint32_t n, int* id, int lane,
                                               int* abort_flag, int* status) {
  const int s = n % kQ;
  if (!warp_wait(&ring->full[s], (n / kQ) & 1, abort_flag, status)) return false;
  *id = *(volatile int*)&ring->id[s];
  __syncwarp();
  if (lane == 0) mbar_arrive(&ring->empty[s]);
  return true;
}

template <int ACT1, int SPEC>
__global__ void __launch_bounds__(kThreads, 1)
    eq_chain_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                       const __grid_constant__ CUtensorMap map_h_store,
                       const __grid_constant__ CUtensorMap map_h_load,
                       const __grid_constant__ CUtensorMap map_y, const uint8_t* __restrict__ w1,
                       const uint8_t* __restrict__ w2, const __half* __restrict__ b1,
                       const __half* __restrict__ b2, ChainInfo ci, int* sync, int* status) {
  static_assert(sizeof(Bars<4>) + sizeof(TaskRing) <= 512, "barrier block");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<4>* bars = reinterpret_cast<Bars<4>*>(smem + S::OFF_BAR);
  TaskRing* ring = reinterpret_cast<TaskRing*>(smem + S::OFF_BAR + 256);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // layer 2 reads H as spectral planes (no transform) or spatially (transformed)
  constexpr bool kL2Planes = SPEC != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::X_ST; ++s) {
      mbar_init(&bars->x_full[s], 1);
      mbar_init(&bars->x_read[s], kXfWarps);
      mbar_init(&bars->x_ready[s], kXfWarps);
      mbar_init(&bars->x_empty[s], 1);
    }
    for (int s = 0; s < S::W_ST; ++s) {
      mbar_init(&bars->w_full[s], 1);
      mbar_init(&bars->w_empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kEpiWarps * 32);
    mbar_init(&bars->drain, 1);
    for (int s = 0; s < kQ; ++s) {
      mbar_init(&ring->full[s], 1);
      mbar_init(&ring->empty[s], kTaskReaders);
    }
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

  if (warp == 0) {
    // ------- X producer and task fetcher -------
    if (lane == 0) {
      int issued_phase[S::X_ST];
      for (int s = 0; s < S::X_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0, n = 0;
      bool ok = true;
      while (ok) {
        const int s = n % kQ;
        if (!(ok = wait_bounded(&ring->empty[s], ((n / kQ) & 1) ^ 1, abort_flag, status))) break;
        const int q = atomicAdd(&sync[0], 1);
        const int id = q < ci.total ? q : -1;
        ring->id[s] = id;
        mbar_arrive(&ring->full[s]);
        ++n;
        if (id < 0) break;
        const Task t = decode(id, ci);
        const int row0 = t.r * BM;
        const int ks_n = t.layer ? ci.ks2 : ci.ks1;
        if (t.layer == 1 &&
            !(ok = wait_row(&sync[2 + t.r], ci.flag_target, abort_flag, status)))
          break;
        for (int ks = 0; ks < ks_n; ++ks, ++it) {
          const int sx = it % S::X_ST;
          const uint32_t ph = (it / S::X_ST) & 1;
          if (!(ok = wait_bounded(&bars->x_empty[sx], ph ^ 1, abort_flag, status))) break;
          mbar_expect_tx(&bars->x_full[sx], X_STAGE_BYTES);
          const uint32_t dst = sbase + S::OFF_X + sx * X_STAGE_BYTES;
          if (t.layer == 0)
            tma_load_3d(dst, &map_x, &bars->x_full[sx], 0, 2 * ks, row0);
          else if (kL2Planes)
            tma_load_3d(dst, &map_h_load, &bars->x_full[sx], S::BK * ks, row0, 0);
          else
            tma_load_3d(dst, &map_h_load, &bars->x_full[sx], 0, 2 * ks, row0);
          issued_phase[sx] = (int)ph;
        }
      }
      if (!ok) {
        for (int s = 0; s < S::X_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->x_full[s], (uint32_t)issued_phase[s]);
      }
    }
  } else if (warp == 2) {
    // ------- weight producer -------
    if (lane == 0) {
      int issued_phase[S::W_ST];
      for (int s = 0; s < S::W_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0, n = 0;
      bool ok = true;
      while (ok) {
        int id;
        if (!(ok = ring_take(ring, n++, &id, abort_flag, status)) || id < 0) break;
        const Task t = decode(id, ci);
        const int ks_n = t.layer ? ci.ks2 : ci.ks1;
        const uint8_t* tiles = t.layer ? w2 : w1;
        for (int ks = 0; ks < ks_n; ++ks, ++it) {
          const int sw = it % S::W_ST;
          const uint32_t ph = (it / S::W_ST) & 1;
          if (!(ok = wait_bounded(&bars->w_empty[sw], ph ^ 1, abort_flag, status))) break;
          mbar_expect_tx(&bars->w_full[sw], S::W_STAGE_BYTES);
          const size_t blob = (size_t)t.j * ks_n + ks;
          bulk_load(sbase + S::OFF_W + sw * S::W_STAGE_BYTES, tiles + blob * S::W_STAGE_BYTES,
                    S::W_STAGE_BYTES, &bars->w_full[sw]);
          issued_phase[sw] = (int)ph;
        }
      }
      if (!ok) {
        for (int s = 0; s < S::W_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->w_full[s], (uint32_t)issued_phase[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tcount = 0, n = 0;
      bool ok = true;
      const uint32_t id_n1 = idesc_f16(BM, BD);
      const uint32_t id_n1_neg = idesc_f16(BM, BD, true);
      const uint32_t id_n2 = idesc_f16(BM, 2 * BD);
      while (ok) {
        int id;
        if (!(ok = ring_take(ring, n++, &id, abort_flag, status)) || id < 0) break;
        const Task t = decode(id, ci);
        const int ks_n = t.layer ? ci.ks2 : ci.ks1;
        const bool planes_in = t.layer == 1 && kL2Planes;
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < ks_n; ++ks, ++it) {
          const int sx = it % S::X_ST, sw = it % S::W_ST;
          uint64_t* xbar = planes_in ? &bars->x_full[sx] : &bars->x_ready[sx];
          if (!(ok = wait_bounded(xbar, (it / S::X_ST) & 1, abort_flag, status))) break;
          if (!(ok = wait_bounded(&bars->w_full[sw], (it / S::W_ST) & 1, abort_flag, status)))
            break;
          tc_fence_after();
          const uint32_t pl = sbase + S::OFF_X + sx * X_STAGE_BYTES;
          const uint32_t wr = sbase + S::OFF_W + sw * S::W_STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < S::KSTEPS; ++kk) {
            const uint32_t ko = 32u * kk;
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            auto A = [&](int p) { return desc_kmajor<S::ROWB>(pl + p * S::PLANE_BYTES + ko); };
            auto B = [&](int p) { return desc_kmajor<S::ROWB>(wr + p * S::WREG_BYTES + ko); };
            umma(tmem + 0, A(0), B(0), id_n1, acc);
            umma(tmem + BD, A(1), B(1), id_n1, acc);
            umma(tmem + 2 * BD, A(2), B(2), id_n2, acc);
            umma(tmem + 2 * BD, A(3), B(3), id_n1_neg, 1u);
            umma(tmem + 3 * BD, A(3), B(2), id_n1, 1u);
          }
          umma_commit(&bars->x_empty[sx]);
          umma_commit(&bars->w_empty[sw]);
        }
        if (ok) umma_commit(&bars->acc_full);
        ++tcount;
      }
      umma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
    // ---------------- epilogue ----------------
    const int q4 = warp & 3;
    const int ch = (warp - kEpiWarp0) >> 2;
    uint8_t* stg = smem + S::OFF_STG + (warp - kEpiWarp0) * kStgBytes;
    __half* bsm = reinterpret_cast<__half*>(smem + S::OFF_BIAS + (warp - kEpiWarp0) * 128);
    uint32_t tcount = 0, n = 0;
    while (true) {
      int id;
      if (!ring_take_warp(ring, n++, &id, lane, abort_flag, status) || id < 0) break;
      const Task t = decode(id, ci);
      const int Cout = t.layer ? ci.C2 : ci.C1;
      const __half* bias = t.layer ? b2 : b1;
      const int64_t row0 = (int64_t)t.r * BM + 32 * q4;
      const int dbase = t.j * BD + (BD / 2) * ch;
      if (2 * lane < BD / 2) {
        const int d = dbase + 2 * lane;
        uint32_t v = 0u;
        if (bias && d < Cout) v = *reinterpret_cast<const uint32_t*>(bias + d);
        reinterpret_cast<uint32_t*>(bsm)[lane] = v;
      }
      __syncwarp();
      if (!warp_wait(&bars->acc_full, tcount & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
      if (t.layer == 0) {
        if constexpr (SPEC)
          epi_slices<4, BD, ACT1, kIoSpectralOut>(lane_addr, ch, lane, stg, bsm, dbase, Cout,
                                                  PlaneStore{&map_h_store, row0, ci.N});
        else
          epi_slices<4, BD, ACT1, kIoSpatial>(lane_addr, ch, lane, stg, bsm, dbase, Cout,
                                              RowStore<4>{&map_h_store, row0, ci.N});
      } else {
        epi_slices<4, BD, 0, kIoSpatial>(lane_addr, ch, lane, stg, bsm, dbase, Cout,
                                         RowStore<4>{&map_y, row0, ci.N});
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
      ++tcount;
      if (t.layer == 0) {
        // this warp's part of the H tile is in memory: count it for the row tile
        if (lane == 0) {
          bulk_wait_all();
          asm volatile("fence.proxy.async.global;" ::: "memory");
          asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(&sync[2 + t.r])
                       : "memory");
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else if (warp >= kXfWarp0) {
    // ---------------- transform (tasks with a spatial input) ----------------
    const int xt = threadIdx.x - kXfWarp0 * 32;
    uint32_t it = 0, n = 0;
    bool ok = true;
    while (ok) {
      int id;
      if (!(ok = ring_take_warp(ring, n++, &id, lane, abort_flag, status)) || id < 0) break;
      const Task t = decode(id, ci);
      const int ks_n = t.layer ? ci.ks2 : ci.ks1;
      if (t.layer == 1 && kL2Planes) {
        it += ks_n;  // the planes arrive ready: keep the ring position in step
        continue;
      }
      for (int ks = 0; ks < ks_n; ++ks, ++it) {
        const int sx = it % S::X_ST;
        if (!(ok = warp_wait(&bars->x_full[sx], (it / S::X_ST) & 1, abort_flag, status))) break;
        uint8_t* slot = smem + S::OFF_X + sx * X_STAGE_BYTES;
        uint4 v[8];
        xf_read<4>(slot, xt, v);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->x_read[sx]);
        if (!(ok = warp_wait(&bars->x_read[sx], (it / S::X_ST) & 1, abort_flag, status))) break;
        xf_write<4>(slot, xt, v);
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
  if (threadIdx.x == 0) {
    // every role of this CTA is done with the counters; the last CTA clears them
    __threadfence();
    if (atomicAdd(&sync[1], 1) == (int)gridDim.x - 1) {
      __threadfence();
      for (int i = 0; i < ci.n_rt; ++i) sync[2 + i] = 0;
      sync[0] = 0;
      __threadfence();
      sync[1] = 0;
    }
  }
}

// Spatial activations [N][channels*4] (FP16) as (64 halves, 128-byte chunk, row).
bool encode_rows(CUtensorMap* m, void* base, int channels, int64_t N, uint32_t box_chunks,
                 uint32_t box_rows) {
  auto encode = encode_fn();
  cuuint64_t dims[3] = {64, (cuuint64_t)channels * 4 / 64, (cuuint64_t)N};
  cuuint64_t strides[2] = {128, (cuuint64_t)channels * 4 * 2};
  cuuint32_t box[3] = {64, box_chunks, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}
// Spectral planes [4][N][channels] (FP16) as (channel, row, plane).
bool encode_planes(CUtensorMap* m, void* base, int channels, int64_t N, uint32_t box_ch,
                   uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto encode = encode_fn();
  cuuint64_t dims[3] = {(cuuint64_t)channels, (cuuint64_t)N, 4};
  cuuint64_t strides[2] = {(cuuint64_t)channels * 2, (cuuint64_t)N * channels * 2};
  cuuint32_t box[3] = {box_ch, box_rows, 4};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int ACT1, int SPEC>
cudaError_t set_chain_attr() {
  return cudaFuncSetAttribute(eq_chain_tc_kernel<ACT1, SPEC>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
}

}  // namespace

size_t chain_tc_sync_bytes(int64_t N) {
  if (N <= 0) return 0;
  return (size_t)(2 + (N + BM - 1) / BM) * sizeof(int);
}

cudaError_t launch_chain_tc(const void* X, int64_t N, int C0, int C1, int C2,
                            const void* W1tiles, const void* b1, const void* W2tiles,
                            const void* b2, void* H, void* Y, int* sync, int* status, int num_sms,
                            int act1, int spectral, cudaStream_t st) {
  if (!fwd_tc_supported(4, DType::F16, N, C0, C1) || !fwd_tc_supported(4, DType::F16, N, C1, C2))
    return cudaErrorNotSupported;
  if (!W1tiles || !W2tiles || !sync) return cudaErrorInvalidValue;
  if (act1 != 0 && act1 != 1) return cudaErrorInvalidValue;
  if (!encode_fn()) return cudaErrorNotSupported;
  CUtensorMap mx, mhs, mhl, my;
  if (!encode_rows(&mx, const_cast<void*>(X), C0, N, 2, BM)) return cudaErrorInvalidValue;
  if (spectral) {
    if (!encode_planes(&mhs, H, C1, N, 16, 32, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !encode_planes(&mhl, H, C1, N, S::BK, BM, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  } else {
    if (!encode_rows(&mhs, H, C1, N, 1, 32) || !encode_rows(&mhl, H, C1, N, 2, BM))
      return cudaErrorInvalidValue;
  }
  if (!encode_rows(&my, Y, C2, N, 1, 32)) return cudaErrorInvalidValue;

  ChainInfo ci;
  ci.N = N;
  ci.C0 = C0; ci.C1 = C1; ci.C2 = C2;
  const int64_t n_rt = (N + BM - 1) / BM;
  ci.n_dt1 = (C1 + BD - 1) / BD;
  ci.n_dt2 = (C2 + BD - 1) / BD;
  if (n_rt * (ci.n_dt1 + ci.n_dt2) > 0x7fffffffLL) return cudaErrorInvalidValue;
  ci.n_rt = (int)n_rt;
  ci.ks1 = (C0 + S::BK - 1) / S::BK;
  ci.ks2 = (C1 + S::BK - 1) / S::BK;
  ci.total = ci.n_rt * (ci.n_dt1 + ci.n_dt2);
  const int grid = ci.total < num_sms ? ci.total : num_sms;
  // at least the first wave takes layer-1 tiles only
  int lag = (3 * ci.n_rt + 2) / 5;
  const int wave = (grid + ci.n_dt1 - 1) / ci.n_dt1;
  if (lag < wave) lag = wave;
  ci.lag = lag < ci.n_rt ? lag : ci.n_rt;
  ci.flag_target = kEpiWarps * ci.n_dt1;

  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = set_chain_attr<0, 0>();
    if (e == cudaSuccess) e = set_chain_attr<1, 0>();
    if (e == cudaSuccess) e = set_chain_attr<0, 1>();
    if (e == cudaSuccess) e = set_chain_attr<1, 1>();
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  auto kernel = spectral ? (act1 ? eq_chain_tc_kernel<1, 1> : eq_chain_tc_kernel<0, 1>)
                         : (act1 ? eq_chain_tc_kernel<1, 0> : eq_chain_tc_kernel<0, 0>);
  kernel<<<grid, kThreads, S::SMEM_BYTES, st>>>(
      mx, mhs, mhl, my, static_cast<const uint8_t*>(W1tiles),
      static_cast<const uint8_t*>(W2tiles), static_cast<const __half*>(b1),
      static_cast<const __half*>(b2), ci, sync, status);
  return cudaGetLastError();
}

}  // namespace eql
