// Host-side launchers shared between the C ABI (eql_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "eql_common.cuh"

namespace eql {

enum class DType { F32 = 0, F16 = 1 };

// Prepared-weight transform: W[D][C][T] -> forward planes [P][D][C] and
// adjoint planes [P][C][D] (see eqlinear.h for the plane order).
cudaError_t launch_prepare(int T, DType dt, const void* W, int C, int D, void* fwd, void* adj,
                           const Twiddles& tw, cudaStream_t st);

// CUDA-core forward over a group-circulant operator.
//   X [N][Cin*T] -> Y [N][Cout*T]; Wt = planes [P][Cin][Cout] of the OTHER block
//   (adjoint block for the forward pass, forward block for dX): the kernel takes
//   Re from the Re planes and Im from the "-Im" slots, which hold the right sign.
// act: output activation (0 none, 1 GELU), applied after the bias.
cudaError_t launch_fwd_simt(int T, DType dt, const void* X, int64_t N, int Cin, int Cout,
                            const void* Wt, const void* bias, void* Y, const Twiddles& tw,
                            int act, cudaStream_t st);

// CUDA-core weight gradient: split reduction over rows into FP32 partial spectra,
// then a finalize kernel (sum in fixed split order, inverse DFT, cast to out_dt).
int wgrad_simt_splits(int T, int64_t N, int C, int D, int num_sms);
size_t wgrad_simt_workspace(int T, int64_t N, int C, int D, int num_sms);
cudaError_t launch_wgrad_simt(int T, DType dt, DType out_dt, const void* X, const void* dY,
                              int64_t N, int C, int D, void* dW, void* dbias, float* ws,
                              int splits, const Twiddles& tw, cudaStream_t st);

// Finalize of a split weight-gradient reduction: partial spectra
// part[split][T planes][D][C] (+ bias partials [split][D]) -> dW[D][C][T], dbias[D]
// in out_dt.
cudaError_t launch_wgrad_finalize(int T, DType out_dt, const float* part, const float* bpart,
                                  int splits, int C, int D, void* dW, void* dbias,
                                  const Twiddles& tw, cudaStream_t st);

// tcgen05/TMEM tensor-core forward for T = 4 and T = 8 (FP16 in, FP32
// accumulate, FP16 out).
// The kernel reads its weights as operand tiles pre-arranged in its own
// shared-memory image (one contiguous blob per out-channel tile and K stage),
// written once by launch_tile_weights from a block of prepared planes.
bool tc_tiles_wanted(int T, DType dt, int C, int D);
size_t tc_tile_bytes(int T, int Cin, int Cout);
cudaError_t launch_tile_weights(int T, const void* planes /* [P][Cout][Cin] */, int Cin,
                                int Cout, void* tiles, cudaStream_t st, int group = 0);
// The dihedral group D4 (T = 8 layout, group = 1): its weight spectrum in the
// tile regions' order, W [D][C][8] -> planes [8][D][C] (FP16).
cudaError_t launch_prepare_d4(const void* W, int C, int D, void* planes, cudaStream_t st);
// Returns cudaErrorNotSupported when the shape does not fit the kernel.
bool fwd_tc_supported(int T, DType dt, int64_t N, int Cin, int Cout);
// drop_w_stage >= 0 is a test-only fault: CTA 0 never issues that weight stage,
// so its bounded waits expire and the kernel reports a timeout.
// io (T = 4 only beyond 0): 0 = spatial X and Y; 1 = Y written as the next
// layer's spectral planes [4][N][Cout] (the group DFT of act(y): X0, X2, Xr, Xi);
// 2 = X read as spectral planes [4][N][Cin] produced that way; 3 = spatial X
// and Y, and X's group spectrum written to `spectrum` [4][N][Cin] (FP16, the
// same planes order), which must be non-null exactly for io = 3.
cudaError_t launch_fwd_tc(int T, const void* X, int64_t N, int Cin, int Cout,
                          const void* Wtiles, const void* bias, void* Y, int* status,
                          int num_sms, int drop_w_stage, int act, int io, cudaStream_t st,
                          int group = 0, void* spectrum = nullptr);

// tcgen05/TMEM tensor-core weight gradient for T = 4, FP16: stream-K over
// (tile, 32-row stage) ranges, FP32 partial slots in `workspace`, then a
// fixed-order finalize (inverse DFT, cast to out_dt: F16 or F32) into
// dW [D][C][4] and dbias [D].  X and dY must be 16-byte aligned (TMA).  N = 0 is
// handled by the caller.
bool wgrad_tc_supported(int T, DType dt, int64_t N, int C, int D, const void* X, const void* dY);
size_t wgrad_tc_workspace(int64_t N, int C, int D, int num_sms);
// planes = 1: X and dY are instead their group spectra as FP16 planes
// [4][N][C] and [4][N][D] (as the forward and dX kernels save them); needs
// C % 64 == 0 and D % 64 == 0 (wgrad_tc_planes_supported).  With plane_rows > N
// the N rows are read from inside planes of plane_rows rows each.  planes = 2:
// the spectra in the tiled layout of the SM-pair kernels (tiled_rows(N) rows per
// 16-channel block, as launch_group_dft_tiled writes them); C, D multiples of 16.
bool wgrad_tc_planes_supported(int64_t N, int C, int D, const void* Xhat, const void* Ghat);
// A convolution's weight gradient in one launch (planes variant): Xs [4][R][C]
// and Gs [4][R][D] are the group spectra of X and dY on the padded pixel grid
// (R rows, planes times 1/4); tap t = i*kw + j multiplies Gs's rows with Xs's
// rows i*wp + j further on, into dW + t*D*C*4 (dW [taps][D][C][4]); dbias once.
// C and D multiples of 64.
size_t wgrad_tc_conv_workspace(int64_t R, int C, int D, int taps, int num_sms);
cudaError_t launch_wgrad_tc_conv(const void* Xs, const void* Gs, int64_t R, int C, int D,
                                 int taps, int kw, int wp, void* workspace, DType out_dt,
                                 void* dW, void* dbias, int* status, int num_sms,
                                 const Twiddles& tw, cudaStream_t st);
cudaError_t launch_wgrad_tc(const void* X, const void* dY, int64_t N, int C, int D,
                            void* workspace, DType out_dt, void* dW, void* dbias, int* status,
                            int num_sms, const Twiddles& tw, cudaStream_t st, int planes = 0,
                            int64_t plane_rows = 0);

// Two chained T = 4 FP16 layers (C0 -> C1 -> C2) in one persistent launch with a
// dynamic tile queue: H = act1(L1(X)) (spatial [N][C1*4], or spectral planes
// [4][N][C1] when `spectral`), Y = L2(H).  `sync` holds chain_tc_sync_bytes(N)
// bytes of counters that must be zero at launch; the kernel leaves them zero.
size_t chain_tc_sync_bytes(int64_t N);
cudaError_t launch_chain_tc(const void* X, int64_t N, int C0, int C1, int C2,
                            const void* W1tiles, const void* b1, const void* W2tiles,
                            const void* b2, void* H, void* Y, int* sync, int* status, int num_sms,
                            int act1, int spectral, cudaStream_t st);

// Group-circulant convolution (T = 4, FP16): X [N][H][W][C*4] -> Y [N][Ho][Wo][D*4],
// KH x KW taps, stride 1, zero padding (ph, pw).  Wtiles: one forward tile block
// (tc_tile_bytes(4, C, D)) per tap, tap-major; planes: conv_tc_planes_bytes of
// scratch for the group DFT of X.
bool conv_tc_supported(int T, DType dt, int64_t N, int H, int W, int C, int D, int KH, int KW,
                       int ph, int pw);
size_t conv_tc_planes_bytes(int64_t N, int H, int W, int C);
cudaError_t launch_conv_tc(const void* X, int64_t N, int H, int W, int C, int D, int KH, int KW,
                           int ph, int pw, const void* Wtiles, const void* bias, void* Y,
                           void* planes, int* status, int num_sms, int act, cudaStream_t st);

// Tiled planes: the group DFT of p4 rows stored as the pair kernel's
// shared-memory operand image (rows padded to a multiple of 128; per plane and
// 16-channel block, 32-byte rows with the 32-byte swizzle; see eql_tc_pair.cu).
int64_t tiled_rows(int64_t N);
size_t tiled_planes_bytes(int64_t N, int channels);
// X [N][C*4] -> tiled planes of X (times 1/4), C a multiple of 16.
cudaError_t launch_group_dft_tiled(const void* X, int64_t N, int C, void* out, cudaStream_t st);

// Pair-CTA (cta_group::2) tensor-core forward for T = 4, FP16, from tiled
// input planes: Y [N][Cout*4] or, with spectral_out, the next layer's tiled
// planes.  Weights: the pair kernel's own stage image (launch_pair_tile_weights
// from a block of prepared planes [5][Cout][Cin]).  Returns
// cudaErrorNotSupported for shapes it does not take (Cin, Cout multiples of 16).
bool pair_tc_supported(int64_t N, int Cin, int Cout);
size_t pair_tile_bytes(int Cin, int Cout);
cudaError_t launch_pair_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                     cudaStream_t st);
cudaError_t launch_pair_tc(const void* Xt, int64_t N, int Cin, int Cout, const void* tiles,
                           const void* bias, void* Y, int* status, int num_sms, int act,
                           int spectral_out, cudaStream_t st);
// Two chained p4 layers on SM pairs (C0 -> C1 -> C2) in one persistent launch
// with a dynamic tile queue: Ht = tiled planes of act1(L1(X)), Y = L2(H) spatial.
// `sync` holds pair_chain_sync_bytes(N) bytes of counters, zero at launch and
// left zero.
size_t pair_chain_sync_bytes(int64_t N);
cudaError_t launch_pair_chain_tc(const void* Xt, int64_t N, int C0, int C1, int C2,
                                 const void* W1tiles, const void* b1, const void* W2tiles,
                                 const void* b2, void* Ht, void* Y, int* sync, int* status,
                                 int num_sms, int act1, cudaStream_t st);

// FP32 p4 layer on SM pairs with 3xTF32 split precision (eql_tc_pair32.cu):
// tiled hi/lo planes of the input (8 planes, 8 FP32 channels per 32-byte row),
// weight stages from prepared FP32 planes [5][Cout][Cin], Y [N][Cout*4] FP32.
// Cin, Cout multiples of 8.
bool pair_tf32_supported(int64_t N, int Cin, int Cout);
size_t tiled_tf32_planes_bytes(int64_t N, int channels);
size_t pair_tf32_tile_bytes(int Cin, int Cout);
cudaError_t launch_pair_tf32_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                          cudaStream_t st);
cudaError_t launch_group_dft_tf32(const void* X, int64_t N, int C, void* out, cudaStream_t st);
cudaError_t launch_pair_tf32(const void* Xt, int64_t N, int Cin, int Cout, const void* tiles,
                             const void* bias, void* Y, int* status, int num_sms, int act,
                             cudaStream_t st);

// Eight-plane layers on SM pairs (eql_tc_pair8.cu): cyclic T = 8 (group 0) and
// the dihedral group D4 (group 1), FP16: tiled planes of the group Fourier
// transform (8 planes, 16 channels per 32-byte row), weight stages from 8
// prepared planes [.][Cout][Cin], Y [N][Cout*8].  Cin, Cout multiples of 16.
bool pair8_supported(int64_t N, int Cin, int Cout);
size_t tiled8_planes_bytes(int64_t N, int channels);
size_t pair8_tile_bytes(int Cin, int Cout);
// d4_adjoint: the dX stages of a D4 layer from its forward planes [8][Cout][Cin]
cudaError_t launch_pair8_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                      cudaStream_t st, int d4_adjoint = 0);
cudaError_t launch_group_dft8_tiled(const void* X, int64_t N, int C, int group, void* out,
                                    cudaStream_t st);
// next_planes = 1: Y is instead the tiled planes (tiled8_planes_bytes(N, Cout))
// of act(Y) for the next layer, as launch_group_dft8_tiled of the spatial output
// (Y rounded to FP16 first); rows N..Np-1 zero.
cudaError_t launch_pair8_tc(const void* Xt, int64_t N, int Cin, int Cout, const void* tiles,
                            const void* bias, void* Y, int* status, int num_sms, int act,
                            int group, cudaStream_t st, int next_planes = 0);

// The group DFT of P pixel rows: X [P][C*4] -> planes [4][P][C] (X0, X2, Xr, Xi,
// each times 1/4; the convolution kernel's pre-pass).
cudaError_t launch_conv_group_planes(const void* X, int64_t P, int C, void* planes,
                                     cudaStream_t st);

// X [N][H][W][c4 halves] moved onto an Ho x Wo pixel grid: out[(n*Ho + oy)*Wo + ox]
// = X[n][oy+i-ph][ox+j-pw] (zero outside the image), c4 a multiple of 8.
cudaError_t launch_conv_shift_rows(const void* X, int64_t N, int H, int W, int c4, int i, int j,
                                   int ph, int pw, int Ho, int Wo, void* out, cudaStream_t st);

// Weight gradient of the D4 layer on CUDA cores (eql_d4_wgrad.cu): FP16 X [N][C*8]
// and dY [N][D*8] -> dW [D][C][8] and dbias [D] in out_dt, through FP32
// partials per row split (d4_wgrad_workspace bytes) summed in a fixed order.
size_t d4_wgrad_workspace(int64_t N, int C, int D, int num_sms);
cudaError_t launch_d4_wgrad(const void* X, const void* dY, int64_t N, int C, int D, DType out_dt,
                            void* dW, void* dbias, float* workspace, int num_sms,
                            cudaStream_t st);

// dst[i] = src[i] rounded to nearest-even in dt (a copy for F32), i < n.
cudaError_t launch_cast_from_f32(DType dt, const float* src, void* dst, int64_t n,
                                 cudaStream_t st);

}  // namespace eql
