// Tensor-core (tcgen05, 3xTF32) variant of the dense back-substitution contraction.
#pragma once
#include "vf_internal.cuh"

namespace vf {

// True when the rows can be fed by a 2-D TMA map: 16-byte aligned rows of a chunk-local buffer,
// or one block of rows shared by all centres whose size is a multiple of the 128-row tile.
// The tensor-core path also needs a relaxation table (it carries the bias in its 4th lane).
bool dense_back_tc_supported(const RowRef& A, Relax rx, long long M, int K, int N, PassGeom pg);
int dense_back_tc_tiles_n(int N);
// Wt_hi / Wt_lo: the node's W transposed to [N, K] (K contiguous) and split into tf32 head and
// fp32 remainder; B = number of centres (rows of rx.P). Same outputs as launch_dense_back, with
// the bias taken from rx.P[.].w; *err is set if a bounded wait expires. test_stall != 0 (tests only)
// withholds one copy in CTA 0 so that its bounded wait expires and the abort path runs.
cudaError_t launch_dense_back_tc(const RowRef& A, Relax rx, const float* Wt_hi, const float* Wt_lo, long long B,
                                 long long M, int K, int N, PassGeom pg, int out_mode, float* out, long long ld_out,
                                 float* cst, const float* centres, float eps, float* part, int* err, int test_stall,
                                 cudaStream_t s);

// Forward product out[M, N] = A[M, K] W^T (+ bias[n]) on the same kernel: W_hi / W_lo hold W in its own
// [N, K] layout (K contiguous) split into tf32 head and fp32 remainder; ident is an identity relaxation row
// ({1, 1, 0, 0}) of at least K entries. A: M rows K floats apart, 16-byte aligned; needs M >= 128.
bool dense_fwd_tc_supported(const float* A, long long M, int K, int N);
cudaError_t launch_dense_fwd_tc(const float* A, long long M, int K, int N, const float* W_hi, const float* W_lo,
                                const float* bias, const float4* ident, float* out, int* err, cudaStream_t s);

}  // namespace vf
