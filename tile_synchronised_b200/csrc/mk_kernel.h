// mk_kernel.h -- host entry points of the device code.
#pragma once
#include <cuda_runtime.h>

#include "mk_internal.h"

namespace mk {
int smem_bytes(const KParams &P);
// Launch the interpreter over P.cta_begin/cta_end; bs = batch rows per GEMV instruction.
cudaError_t launch_step(const KParams &P, int bs, int n_ctas, cudaStream_t s, bool cooperative, bool pdl_attr);
const void *step_kernel_func(const KParams &P);
cudaError_t launch_pack(const void *src, const void *src2, void *dst, int n_rows, int k, int kc, int nkb, int tiles,
                        int rows, int mode, cudaStream_t s);
cudaError_t launch_set_position(State *state, int pos, cudaStream_t s);
// Fused SwiGLU first stage (fp16): variant MK_SWIGLU_ROW or MK_SWIGLU_COL.
cudaError_t launch_swiglu(const void *x, const void *wg, const void *wu, void *out, int B, int K, int N, int variant,
                          cudaStream_t s);
// The same stage on the tcgen05 tensor cores (K a multiple of 128, N of 128; B <= 128).
bool swiglu_tc_supported(int B, int K, int N);
// The column tiling on the same TMA pipeline, CUDA cores (B <= 8, N % 128 == 0).
bool swiglu_col_tma_supported(int B, int K, int N);
cudaError_t launch_swiglu_col_tma(const void *x, const void *wg, const void *wu, void *out, int B, int K, int N,
                                  cudaStream_t s);
cudaError_t launch_swiglu_tc(const void *x, const void *wg, const void *wu, void *out, int B, int K, int N,
                             cudaStream_t s);
// Last error of a context-free call (the isolated operations) on this thread.
void set_op_error(const char *msg);
const char *op_error();
}  // namespace mk
