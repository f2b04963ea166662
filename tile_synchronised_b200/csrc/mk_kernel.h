// mk_kernel.h -- host entry points of the device code.
#pragma once
#include <cuda_runtime.h>

#include <string>

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
// Split-KV decode attention whose attended length is read from device memory
// (mk_attn.cu); the caller has checked the shapes.
cudaError_t launch_attention_dev(const float *q, const void *k, const void *v, int B, int nq, int nkv, int d,
                                 int max_seq, const int *n_pos_dev, int chunks, float *out, float *part,
                                 cudaStream_t s);
// y[b][m] = sum_k W[m][k] x[b][k] on the tensor cores (mk_linear_tc.cu) with W
// one of the megakernel's packed matrices, [tiles][K / kc][rows][kc] bf16, and
// x bf16 [B][K] (K = the packed width, zero past the logical one).
cudaError_t launch_linear_tc_packed(const void *x, const void *w, float *y, int B, int K, int M, int kc, int rows,
                                    cudaStream_t s, bool pdl = false);
// The same as a stream-K launch when the tiles would not fill the SMs evenly
// (mk_linear_tc.cu): ws holds kSkWorkspaceFloats floats and flags
// kSkWorkspaceFlags words, zero before the first launch (every launch leaves
// them zero); falls back to the launch above otherwise.
constexpr size_t kSkWorkspaceFloats = (size_t)256 * 256 * 128;
constexpr size_t kSkWorkspaceFlags = 256;
cudaError_t launch_linear_tc_packed_sk(const void *x, const void *w, float *y, int B, int K, int M, int kc, int rows,
                                       float *ws, uint32_t *flags, cudaStream_t s, bool pdl);
// Causal attention of prefill rows (mk_attn.cu): row r of q / out attends
// positions 0 .. row_len[r] - 1 of sequence row_seq[r] of one layer's cache.
// With `hilo` set, the output goes there instead of `out`, as the bf16 pair
// hi = bf16(o), lo = bf16(o - hi) in rows r and rows + r (ld columns apart,
// ld = nq * d): the tensor cores' input form.
cudaError_t launch_attention_rows(const float *q, const void *k, const void *v, int rows, int nq, int nkv, int d,
                                  int max_seq, const int *row_seq, const int *row_len, int chunks, float *out,
                                  float *part, cudaStream_t s, bool pdl = false, void *hilo = nullptr);
// The tensor-core prefill of a megakernel context (mk_tcdec.cu): positions
// 0 .. T-1 of every sequence through the decoder in chunks of kPrefillRows,
// every projection one tensor-core GEMM over the packed weights.  Fills the KV
// cache only.
struct PrefillTc {
    int L, H, nq, nkv, d, I, V, B, max_seq, qk_norm;
    float eps;
    double theta;
    const void *embed;
    const LayerW *layers;  // host array of the L layers' device pointers
    PackedMat qkv, o, gu, down, lm;  // the packed matrices' geometry
    const void *lm_w, *final_norm;  // the packed LM head and the final norm gains
    uint16_t *kcache, *vcache;
    State *state;
    uint8_t *scratch;
    size_t scratch_bytes;
};
size_t prefill_scratch_bytes(int H, int nq, int d, int kmax, int mmax);
// Returns an empty string, or the reason it stopped.
std::string prefill_tc(const PrefillTc &a, const int32_t *tokens, int T, cudaStream_t s);
// One decode step of every sequence at the context's current position (read
// on the device from a.state, then advanced) through the same row pass, plus
// the final norm, the LM head and the argmax: the megakernel's step on the
// tensor cores.  tokens [B] in; next [B] (and logits [B][V] if set) out.
std::string decode_tc(const PrefillTc &a, const int32_t *tokens, int32_t *next, float *logits, cudaStream_t s);
// The scratch's own token and argmax rows (a captured step copies through them).
int32_t *decode_tc_tokens(const PrefillTc &a);
int32_t *decode_tc_next(const PrefillTc &a);
// Last error of a context-free call (the isolated operations) on this thread.
void set_op_error(const char *msg);
const char *op_error();
}  // namespace mk
