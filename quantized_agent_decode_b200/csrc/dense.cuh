// dense.cuh -- the prefill-chunk (dense, tcgen05) quantized GEMM launch interface.
#pragma once
#include "gemm.cuh"

namespace qad {

// Workspace: the fp16 activation tiles (M padded to 256) plus the row scales.
size_t dense_ws_bytes(int K, int M);
int dense_set_stall(int at);  // test hook behind qad_debug_stall (kernel 1)
int make_dense_maps(int fmt, const void *W, int N, int K, WeightMapsBlob *out);
// Y[M][N] fp32 (overwritten) = X[M][K] bf16 times the quantized weights^T.
int launch_dense(int fmt, const void *W, int N, int K, const uint16_t *X, int M, float *Y, void *ws, cudaStream_t s);

}  // namespace qad
