// mk_tcdec.cu -- a batched decode step whose projections run on the tcgen05
// tensor cores: every matrix of the decoder (QKV, O, gate, up, down, LM head)
// goes through mk_linear_tc, which reads each weight byte once for the whole
// batch, and the attention through the split-KV kernels of mk_attn.cu.  The
// rest of the step is small kernels over [batch, width] rows: the embedding
// gather, RMSNorm, qk-norm + RoPE + KV append, the residual adds, SiLU * up,
// and the LM head's argmax.
//
// Precision.  The MMA takes bf16 operands; a row rounded to bf16 loses 8 bits
// of every activation, which over a deep decoder moves the logits by ~1-2 % of
// their range.  So every activation row x enters as two bf16 rows, hi =
// bf16(x) and lo = bf16(x - hi), in batch positions b and B + b of the
// projection's input, and the output of row b is y[b] + y[B + b]: about 16
// significant bits per activation for twice the MMA work, on a tensor pipe
// that these shapes leave mostly idle.
//
// The math is the plain decoder step (the one the megakernel computes): for
// each layer, h = RMSNorm(x) * g1; q, k, v = h W_q^T, h W_k^T, h W_v^T;
// optional per-head RMSNorm of q and k; rotate-half RoPE at the position;
// append k, v to the cache; attention over positions 0 .. pos; x += o W_o^T;
// h = RMSNorm(x) * g2; x += (SiLU(h W_g^T) * (h W_u^T)) W_d^T; then the
// logits of RMSNorm(x) * g_f and their argmax, lowest index on ties.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_device.cuh"
#include "mk_kernel.h"

namespace mk {
namespace tcdec {

constexpr int kRowThreads = 256;
constexpr int kArgmaxThreads = 512;
constexpr int kArgParts = 32;     // slices of a row's logits in the first argmax pass (one warp reduces them)
constexpr int kNormThreads = 1024;
constexpr int kNormPer = 8;       // RMSNorm rows up to kNormThreads * kNormPer = 8192 wide
constexpr int kMaxBatch = 32;      // 2 * batch rows must fit mk_linear_tc's 64
constexpr int kMaxChunks = 64;     // the split-KV chunk count never exceeds this

__device__ __forceinline__ void put_hilo(__nv_bfloat16 *hi, __nv_bfloat16 *lo, float v) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    *hi = h;
    *lo = __float2bfloat16_rn(v - __bfloat162float(h));
}

// Sum over the block (blockDim.x a multiple of 32, at most 1024).
__device__ float block_sum(float v, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (int)blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    __syncthreads();  // red may still be read by a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float s = 0.f;
    for (int w = 0; w < nw; ++w) s += red[w];
    return s;
}

// x[b][:] = E[tok[b]][:]; an out-of-range token leaves the row at zero and
// sets the status word.
__global__ void embed_kernel(const int32_t *tok, const uint16_t *E, float *x, int H, int V, int *status) {
    const int b = blockIdx.x, t = tok[b];
    const bool ok = t >= 0 && t < V;
    if (!ok && threadIdx.x == 0) atomicOr(status, 1);
    for (int i = threadIdx.x; i < H; i += blockDim.x) x[(size_t)b * H + i] = ok ? bf2f(E[(size_t)t * H + i]) : 0.f;
}

// out rows b (hi) and B + b (lo) = RMSNorm(x[b]) * g, epsilon inside the root.
__global__ void norm_hilo_kernel(const float *x, const uint16_t *g, __nv_bfloat16 *out, int B, int H, float eps) {
    __shared__ float red[32];
    const int b = blockIdx.x;
    const float *xr = x + (size_t)b * H;
    float ss = 0.f;
    for (int i = threadIdx.x; i < H; i += blockDim.x) ss = fmaf(xr[i], xr[i], ss);
    ss = block_sum(ss, red);
    const float r = rsqrtf(ss / (float)H + eps);
    for (int i = threadIdx.x; i < H; i += blockDim.x)
        put_hilo(out + (size_t)b * H + i, out + (size_t)(B + b) * H + i, xr[i] * r * bf2f(g[i]));
}

// One block per (head, sequence), head_dim threads.  Heads 0 .. nq-1 are q,
// then nkv k heads, then nkv v heads; y* hold the hi and lo rows of each
// projection.  q and k get the optional per-head RMSNorm and the RoPE
// rotation (pairs i, i + d/2, angle pos * theta^(-2i/d) in double); q goes to
// q_out, k and v to the layer's cache at `pos` as bf16.  The position is read
// from device memory (posw[0]), so a captured step replays at any position.
__global__ void qkv_post_kernel(const float *yq, const float *yk, const float *yv, int B, int nq, int nkv, int d,
                                const uint16_t *qn, const uint16_t *kn, int qk_norm, float eps, double theta,
                                const int *posw, float *q_out, uint16_t *kc, uint16_t *vc, int max_seq) {
    extern __shared__ float buf[];  // d values, then 32 partial sums
    float *red = buf + d;
    const int head = blockIdx.x, b = blockIdx.y, i = threadIdx.x;
    const int pos = posw[0];
    const float *src;
    int M, off;
    if (head < nq) {
        src = yq;
        M = nq * d;
        off = head * d;
    } else if (head < nq + nkv) {
        src = yk;
        M = nkv * d;
        off = (head - nq) * d;
    } else {
        src = yv;
        M = nkv * d;
        off = (head - nq - nkv) * d;
    }
    float v = src[(size_t)b * M + off + i] + src[(size_t)(B + b) * M + off + i];
    const int g = head < nq ? 0 : (head < nq + nkv ? head - nq : head - nq - nkv);
    const size_t crow = (((size_t)b * nkv + g) * max_seq + pos) * d;
    if (head >= nq + nkv) {
        vc[crow + i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        return;
    }
    if (qk_norm) {
        const float ss = block_sum(v * v, red);
        v = v * rsqrtf(ss / (float)d + eps) * bf2f((head < nq ? qn : kn)[i]);
    }
    buf[i] = v;
    __syncthreads();
    const int h2 = d / 2, j = i < h2 ? i : i - h2;
    const double ang = (double)pos * pow(theta, -2.0 * (double)j / (double)d);
    double sd, cd;
    sincos(ang, &sd, &cd);
    const float c = (float)cd, s = (float)sd;
    const float r = i < h2 ? buf[i] * c - buf[i + h2] * s : buf[i] * c + buf[i - h2] * s;
    if (head < nq)
        q_out[((size_t)b * nq + head) * d + i] = r;
    else
        kc[crow + i] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
}

// out rows b, B + b = hi / lo of a[b][:] (n values per row).
__global__ void cast_hilo_kernel(const float *a, __nv_bfloat16 *out, int B, int n) {
    const int b = blockIdx.y;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        put_hilo(out + (size_t)b * n + i, out + (size_t)(B + b) * n + i, a[(size_t)b * n + i]);
}

// x[b][i] += y[b][i] + y[B + b][i]
__global__ void residual_add_kernel(float *x, const float *y, int B, int H) {
    const int b = blockIdx.y;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < H; i += gridDim.x * blockDim.x)
        x[(size_t)b * H + i] += y[(size_t)b * H + i] + y[(size_t)(B + b) * H + i];
}

// out rows b, B + b = hi / lo of SiLU(g) * u, g and u summed from their hi and
// lo rows.
__global__ void swiglu_hilo_kernel(const float *yg, const float *yu, __nv_bfloat16 *out, int B, int I) {
    const int b = blockIdx.y;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < I; j += gridDim.x * blockDim.x) {
        const float g = yg[(size_t)b * I + j] + yg[(size_t)(B + b) * I + j];
        const float u = yu[(size_t)b * I + j] + yu[(size_t)(B + b) * I + j];
        put_hilo(out + (size_t)b * I + j, out + (size_t)(B + b) * I + j, g / (1.0f + expf(-g)) * u);
    }
}

// posw[0] = the position of the step, posw[1] = the attended length.
__global__ void set_pos_kernel(int *posw, int pos) {
    posw[0] = pos;
    posw[1] = pos + 1;
}

// One block per sequence: logits[b][v] = y[b][v] + y[B + b][v] (written when
// `logits` is set) and next[b] = their argmax, lowest index on ties.  With no
// finite logit to pick (a projection that gave up writes NaN), next[b] is set
// to 0, a valid token, and bit 2 of the status word is set.
__global__ void lm_argmax_kernel(const float *y, float *logits, int32_t *next, int B, int V, int *status) {
    __shared__ float bv_s[32];
    __shared__ int bi_s[32];
    const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int v = threadIdx.x; v < V; v += blockDim.x) {
        const float l = y[(size_t)b * V + v] + y[(size_t)(B + b) * V + v];
        if (logits) logits[(size_t)b * V + v] = l;
        if (l > bv || (l == bv && v < bi)) {
            bv = l;
            bi = v;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
        }
    }
    if (lane == 0) {
        bv_s[warp] = bv;
        bi_s[warp] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            if (bv_s[w] > bv_s[0] || (bv_s[w] == bv_s[0] && bi_s[w] < bi_s[0])) {
                bv_s[0] = bv_s[w];
                bi_s[0] = bi_s[w];
            }
        if (bi_s[0] == 0x7fffffff) {
            atomicOr(status, 2);
            bi_s[0] = 0;
        }
        next[b] = bi_s[0];
    }
}

// ------------------------------------------------------------------ prefill rows
// Every kernel of the row pass is launched with programmatic dependent launch:
// it first waits for the kernel before it (griddepcontrol.wait: that kernel
// has finished and its writes are visible), then lets the next one launch, so
// the next kernel's launch and set-up overlap this one.  Without the launch
// attribute both instructions return at once.
__device__ __forceinline__ void row_pass_prologue() {
    pdl_wait();
    pdl_launch_dependents();
}

// Launch `k` on `s` with programmatic dependent launch allowed.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...);
}
// The prefill of a megakernel context on the tensor cores: R <= 128
// consecutive positions t0 .. t0 + R - 1 of one sequence b go through the
// decoder together, every projection one mk_linear_tc call over the
// context's packed weights (which are plain row-major [rows, kc] matrices
// when each has a single K block), activations as hi/lo bf16 row pairs as in
// the batched step, and attention causal per row (position t0 + r attends to
// 0 .. t0 + r).  Only the KV cache is kept: the last layer stops after its
// K/V rows.

// x[r][:] = E[tok][:] with tok = tok[b * tok_stride + t0 + r] (a prefill
// chunk: positions t0 + r of sequence b) or, for b < 0, tok[r] of sequence r
// (a decode step); a token outside [0, V) decodes from token 0 and is
// recorded in the context's state (first one wins), as the megakernel does.
__global__ void prefill_embed_kernel(const int32_t *tok, int64_t tok_stride, int b, int t0, const uint16_t *E,
                                     float *x, int H, int V, State *state, int seq0) {
    row_pass_prologue();
    const int r = blockIdx.x;
    const int seq = b < 0 ? seq0 + r : b;
    int t = b < 0 ? tok[r] : tok[(int64_t)b * tok_stride + t0 + r];
    if (t < 0 || t >= V) {
        if (threadIdx.x == 0 && atomicCAS(&state->tok_err, 0u, (uint32_t)seq + 1u) == 0u) state->tok_bad = t;
        t = 0;
    }
    for (int i = threadIdx.x; i < H; i += blockDim.x) x[(size_t)r * H + i] = bf2f(E[(size_t)t * H + i]);
}

// x[r] += y[r][:H] + y[R + r][:H] when y is given (the residual add of a
// projection's hi and lo outputs, y rows M wide), then out rows r and R + r
// (Kp wide) = hi / lo of RMSNorm(x[r]) * g, zero past H.  One block per row
// with the whole row in registers (H <= kNormThreads * kNormPer): every load
// of the row is in flight at once, and x is read and written once.
__global__ void __launch_bounds__(kNormThreads) residual_norm_kernel(float *x, const float *y, int M,
                                                                     const uint16_t *g, __nv_bfloat16 *out, int R,
                                                                     int H, int Kp, float eps) {
    row_pass_prologue();
    __shared__ float red[32];
    const int r = blockIdx.x, t = threadIdx.x;
    float *xr = x + (size_t)r * H;
    float v[kNormPer];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
        const int i = t + j * kNormThreads;
        float xv = 0.f;
        if (i < H) {
            xv = xr[i];
            if (y) xv += y[(size_t)r * M + i] + y[(size_t)(R + r) * M + i];
        }
        v[j] = xv;
        ss = fmaf(xv, xv, ss);
    }
    if (y)
#pragma unroll
        for (int j = 0; j < kNormPer; ++j)
            if (t + j * kNormThreads < H) xr[t + j * kNormThreads] = v[j];
    ss = block_sum(ss, red);
    const float rs = rsqrtf(ss / (float)H + eps);
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
        const int i = t + j * kNormThreads;
        if (i < Kp) put_hilo(out + (size_t)r * Kp + i, out + (size_t)(R + r) * Kp + i, i < H ? v[j] * rs * bf2f(g[i]) : 0.f);
    }
    for (int i = t + kNormPer * kNormThreads; i < Kp; i += kNormThreads)
        put_hilo(out + (size_t)r * Kp + i, out + (size_t)(R + r) * Kp + i, 0.f);
}

// One block per (head, row), head_dim threads, over the packed QKV output y
// [2R][M] (q heads, then k, then v): the optional per-head RMSNorm and RoPE at
// the row's position row_len[r] - 1; q to q_out [R][nq][d], k and v to the
// layer's cache rows of sequence row_seq[r] at that position.
__global__ void prefill_qkv_kernel(const float *y, int R, int M, int nq, int nkv, int d, const uint16_t *qn,
                                   const uint16_t *kn, int qk_norm, float eps, double theta, const int *row_seq,
                                   const int *row_len, float *q_out, uint16_t *kc, uint16_t *vc, int max_seq) {
    row_pass_prologue();
    extern __shared__ float buf[];
    float *red = buf + d;
    const int head = blockIdx.x, r = blockIdx.y, i = threadIdx.x;
    const int b = row_seq[r], pos = row_len[r] - 1;
    float v = y[(size_t)r * M + head * d + i] + y[(size_t)(R + r) * M + head * d + i];
    const int g = head < nq ? 0 : (head < nq + nkv ? head - nq : head - nq - nkv);
    const size_t crow = (((size_t)b * nkv + g) * max_seq + pos) * d;
    if (head >= nq + nkv) {
        vc[crow + i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        return;
    }
    if (qk_norm) {
        const float ss = block_sum(v * v, red);
        v = v * rsqrtf(ss / (float)d + eps) * bf2f((head < nq ? qn : kn)[i]);
    }
    buf[i] = v;
    __syncthreads();
    const int h2 = d / 2, j = i < h2 ? i : i - h2;
    const double ang = (double)pos * pow(theta, -2.0 * (double)j / (double)d);
    double sd, cd;
    sincos(ang, &sd, &cd);
    const float c = (float)cd, sn = (float)sd;
    const float o = i < h2 ? buf[i] * c - buf[i + h2] * sn : buf[i] * c + buf[i - h2] * sn;
    if (head < nq)
        q_out[((size_t)r * nq + head) * d + i] = o;
    else
        kc[crow + i] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
}

// row_seq[r] = b, row_len[r] = t0 + r + 1: the rows' sequence and attended
// length (a prefill chunk); for b < 0, row r is sequence r at the context's
// current position (a decode step; read on the device, so a captured step
// replays at any position).  Also clears the stream-K projections' flags
// (left zero by every launch that completes; this heals a pass after one
// that gave up).
__global__ void prefill_rows_kernel(int *row_seq, int *row_len, int R, int b, int t0, const State *state, int seq0,
                                    uint32_t *sk_flags) {
    row_pass_prologue();
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
        row_seq[r] = b < 0 ? seq0 + r : b;
        row_len[r] = b < 0 ? state->pos + 1 : t0 + r + 1;
    }
    for (int i = threadIdx.x; i < (int)kSkWorkspaceFlags; i += blockDim.x) sk_flags[i] = 0u;
}

// The argmax of each row's logits y[r] + y[n + r] (hi and lo outputs, ldy
// apart), lowest index on ties, NaN never chosen, in two passes: block (p, r)
// reduces the p-th of kArgParts slices of row r (and copies its logits out
// when asked), then argmax_final_kernel reduces the slices' winners.  The
// rule is a total order on (value, index), so the result does not depend on
// the order of the reductions.
__device__ __forceinline__ void arg_better(float &bv, int &bi, float ov, int oi) {
    if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
    }
}

__global__ void __launch_bounds__(kArgmaxThreads) argmax_part_kernel(const float *y, int ldy, int n, float *logits,
                                                                     int V, int seq0, float *pv, int *pi) {
    row_pass_prologue();
    __shared__ float bv_s[32];
    __shared__ int bi_s[32];
    const int p = blockIdx.x, r = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int v0 = (int)((long long)p * V / kArgParts), v1 = (int)((long long)(p + 1) * V / kArgParts);
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int base = v0 + (int)threadIdx.x; base < v1; base += 4 * kArgmaxThreads) {
        float l[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int v = base + u * kArgmaxThreads;
            l[u] = v < v1 ? y[(size_t)r * ldy + v] + y[(size_t)(n + r) * ldy + v] : -INFINITY;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int v = base + u * kArgmaxThreads;
            if (v < v1) {
                if (logits) logits[(size_t)(seq0 + r) * V + v] = l[u];
                arg_better(bv, bi, l[u], v);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        arg_better(bv, bi, __shfl_xor_sync(0xFFFFFFFFu, bv, o), __shfl_xor_sync(0xFFFFFFFFu, bi, o));
    if (lane == 0) {
        bv_s[warp] = bv;
        bi_s[warp] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kArgmaxThreads / 32; ++w) arg_better(bv, bi, bv_s[w], bi_s[w]);
        pv[r * kArgParts + p] = bv;
        pi[r * kArgParts + p] = bi;
    }
}

// One warp per row over its kArgParts slice winners; a row without a finite
// or infinite logit (all NaN) decodes token 0 and sets the state's error.
__global__ void argmax_final_kernel(const float *pv, const int *pi, int32_t *next, int seq0, State *state) {
    row_pass_prologue();
    const int r = blockIdx.x, lane = threadIdx.x;
    float bv = pv[r * kArgParts + lane];
    int bi = pi[r * kArgParts + lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        arg_better(bv, bi, __shfl_xor_sync(0xFFFFFFFFu, bv, o), __shfl_xor_sync(0xFFFFFFFFu, bi, o));
    if (lane == 0) {
        if (bi == 0x7fffffff) {
            atomicCAS(&state->err, 0u, 5u);
            bi = 0;
        }
        next[seq0 + r] = bi;
    }
}

// After a decode step on the tensor cores: the context's position advances.
__global__ void advance_pos_kernel(State *state) {
    row_pass_prologue();
    state->pos += 1;
}

// out rows r, R + r (Kp wide) = hi / lo of a[r][0 .. n), zero past n.
__global__ void prefill_cast_kernel(const float *a, __nv_bfloat16 *out, int R, int n, int Kp) {
    row_pass_prologue();
    const int r = blockIdx.y;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < Kp; i += gridDim.x * blockDim.x)
        put_hilo(out + (size_t)r * Kp + i, out + (size_t)(R + r) * Kp + i, i < n ? a[(size_t)r * n + i] : 0.f);
}

// The packed gate/up output y [2R][M] interleaves them tile by tile: packed
// row t*rows + k is gate row t*rows/2 + k for k < rows/2, else up row
// t*rows/2 + k - rows/2.  out rows r, R + r (Kp wide) = hi / lo of
// SiLU(gate) * up, zero past I.
__global__ void prefill_swiglu_kernel(const float *y, __nv_bfloat16 *out, int R, int I, int M, int rows, int Kp) {
    row_pass_prologue();
    const int r = blockIdx.y, half = rows / 2;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < Kp; j += gridDim.x * blockDim.x) {
        float val = 0.f;
        if (j < I) {
            const size_t gi = (size_t)(j / half) * rows + j % half, ui = gi + half;
            const float gt = y[(size_t)r * M + gi] + y[(size_t)(R + r) * M + gi];
            const float up = y[(size_t)r * M + ui] + y[(size_t)(R + r) * M + ui];
            val = gt / (1.0f + expf(-gt)) * up;
        }
        put_hilo(out + (size_t)r * Kp + j, out + (size_t)(R + r) * Kp + j, val);
    }
}

// Byte offsets of the workspace pieces (each 256-byte aligned).
struct Layout {
    size_t x, h, yq, yk, yv, ya, yg, yu, ylm, q, attn, scratch, scratch_bytes, status, tok, nxt, posw, lg, total;
};

static Layout layout(const mk_config &c) {
    Layout o{};
    const size_t B = (size_t)c.batch, H = (size_t)c.hidden, I = (size_t)c.intermediate, V = (size_t)c.vocab;
    const size_t QD = (size_t)c.n_heads * c.head_dim, KD = (size_t)c.n_kv_heads * c.head_dim;
    const size_t kmax = std::max(H, std::max(QD, I));
    size_t at = 0;
    auto take = [&](size_t bytes) {
        const size_t p = at;
        at += (bytes + 255) / 256 * 256;
        return p;
    };
    o.x = take(B * H * 4);
    o.h = take(2 * B * kmax * 2);
    o.yq = take(2 * B * QD * 4);
    o.yk = take(2 * B * KD * 4);
    o.yv = take(2 * B * KD * 4);
    o.ya = take(2 * B * H * 4);
    o.yg = take(2 * B * I * 4);
    o.yu = take(2 * B * I * 4);
    o.ylm = take(2 * B * V * 4);
    o.q = take(B * QD * 4);
    o.attn = take(B * QD * 4);
    o.scratch_bytes = mk_attention_scratch_bytes(c.batch, c.n_heads, c.head_dim, kMaxChunks);
    o.scratch = take(o.scratch_bytes);
    o.status = take(4);
    o.tok = take(B * 4);   // the step's tokens, copied in from the caller
    o.nxt = take(B * 4);   // its argmax, copied out to the caller
    o.posw = take(8);      // position and attended length
    o.lg = take(B * V * 4);  // its logits, copied out when the caller asks for them
    o.total = at;
    return o;
}

}  // namespace tcdec

size_t prefill_scratch_bytes(int H, int nq, int d, int kmax, int mmax) {
    const size_t R = kPrefillRows;
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    return up(R * H * 4) + up(2 * R * kmax * 2) + up(2 * R * (size_t)mmax * 4) + 2 * up(R * nq * d * 4) +
           up(R * nq * kPrefillChunks * (size_t)(d + 2) * 4) + up(2 * R * 4) + 2 * up(64 * 4) +
           up(kSkWorkspaceFloats * 4) + up(kSkWorkspaceFlags * 4);
}

namespace {

// The row pass's buffers, carved out of the context's scratch region.
struct RowsScratch {
    float *x, *y, *q, *attn, *part;
    __nv_bfloat16 *h;
    int *rows;           // row_seq [kPrefillRows], then row_len [kPrefillRows]
    int32_t *tok, *nxt;  // a decode step's tokens and argmax (64 each)
    float *skws;         // the stream-K projections' contributions
    uint32_t *skflags;   // and their flags
};

int pk(const PackedMat &m) { return m.nkb * m.kc; }    // a packed matrix's width as a GEMM operand
int pm(const PackedMat &m) { return m.tiles * m.rows; }  // and its height

bool carve(const PrefillTc &a, RowsScratch &sc) {
    const int R = kPrefillRows;
    const int kmax = std::max(std::max(pk(a.qkv), pk(a.o)), std::max(pk(a.gu), std::max(pk(a.down), pk(a.lm))));
    const int mmax = std::max(std::max(pm(a.qkv), pm(a.o)), std::max(pm(a.gu), std::max(pm(a.down), pm(a.lm))));
    if (a.scratch_bytes < prefill_scratch_bytes(a.H, a.nq, a.d, kmax, mmax)) return false;
    uint8_t *p = a.scratch;
    auto take = [&](size_t bytes) {
        uint8_t *q = p;
        p += (bytes + 255) / 256 * 256;
        return q;
    };
    sc.x = reinterpret_cast<float *>(take((size_t)R * a.H * 4));
    sc.h = reinterpret_cast<__nv_bfloat16 *>(take((size_t)2 * R * kmax * 2));
    sc.y = reinterpret_cast<float *>(take((size_t)2 * R * mmax * 4));
    sc.q = reinterpret_cast<float *>(take((size_t)R * a.nq * a.d * 4));
    sc.attn = reinterpret_cast<float *>(take((size_t)R * a.nq * a.d * 4));
    sc.part = reinterpret_cast<float *>(take((size_t)R * a.nq * kPrefillChunks * (a.d + 2) * 4));
    sc.rows = reinterpret_cast<int *>(take((size_t)2 * R * 4));
    sc.tok = reinterpret_cast<int32_t *>(take(64 * 4));
    sc.nxt = reinterpret_cast<int32_t *>(take(64 * 4));
    sc.skws = reinterpret_cast<float *>(take(kSkWorkspaceFloats * 4));
    sc.skflags = reinterpret_cast<uint32_t *>(take(kSkWorkspaceFlags * 4));
    return true;
}

// n rows (their sequence and attended length in sc.rows, their embeddings in
// sc.x) through every layer; without `full` the last layer stops after its
// K/V rows (a prefill keeps only the cache).
std::string rows_through_layers(const PrefillTc &a, const RowsScratch &sc, int n, int chunks, bool full,
                                cudaStream_t s) {
    using namespace tcdec;
    const int R = kPrefillRows;
    const size_t layer_elems = (size_t)a.B * a.nkv * a.max_seq * a.d;
    std::string err;
    auto lin = [&](const void *w, const PackedMat &m) {
        if (!err.empty()) return;
        const cudaError_t e =
            launch_linear_tc_packed_sk(sc.h, w, sc.y, 2 * n, pk(m), pm(m), m.kc, m.rows, sc.skws, sc.skflags, s, true);
        if (e != cudaSuccess) err = std::string("projection: ") + cudaGetErrorString(e);
    };
    for (int l = 0; l < a.L && err.empty(); ++l) {
        const LayerW &W = a.layers[l];
        uint16_t *kc = a.kcache + (size_t)l * layer_elems, *vc = a.vcache + (size_t)l * layer_elems;
        if (l == 0)  // later layers get their normalised input from the previous layer's last residual add
            launch_pdl(residual_norm_kernel, dim3(n), dim3(kNormThreads), 0, s, sc.x, static_cast<const float *>(nullptr),
                       0, static_cast<const uint16_t *>(W.attn_norm), sc.h, n, a.H, pk(a.qkv), a.eps);
        lin(W.qkv, a.qkv);
        if (!err.empty()) break;
        launch_pdl(prefill_qkv_kernel, dim3((unsigned)(a.nq + 2 * a.nkv), (unsigned)n), dim3(a.d),
                   (a.d + 32) * sizeof(float), s, sc.y, n, pm(a.qkv), a.nq, a.nkv, a.d,
                   static_cast<const uint16_t *>(W.q_norm), static_cast<const uint16_t *>(W.k_norm), a.qk_norm, a.eps,
                   a.theta, sc.rows, sc.rows + R, sc.q, kc, vc, a.max_seq);
        if (!full && l == a.L - 1) break;  // a prefill keeps only the cache: the last layer ends at its K/V
        // the attention output goes straight into the O projection's hi / lo
        // input rows when their width is the logical one (no padding to clear)
        const bool direct = pk(a.o) == a.nq * a.d;
        const cudaError_t e = launch_attention_rows(sc.q, kc, vc, n, a.nq, a.nkv, a.d, a.max_seq, sc.rows,
                                                    sc.rows + R, chunks, sc.attn, sc.part, s, true,
                                                    direct ? static_cast<void *>(sc.h) : nullptr);
        if (e != cudaSuccess) {
            err = std::string("attention: ") + cudaGetErrorString(e);
            break;
        }
        if (!direct)
            launch_pdl(prefill_cast_kernel, dim3(8, (unsigned)n), dim3(kRowThreads), 0, s, sc.attn, sc.h, n,
                       a.nq * a.d, pk(a.o));
        lin(W.o, a.o);
        launch_pdl(residual_norm_kernel, dim3(n), dim3(kNormThreads), 0, s, sc.x, static_cast<const float *>(sc.y),
                   pm(a.o), static_cast<const uint16_t *>(W.mlp_norm), sc.h, n, a.H, pk(a.gu), a.eps);
        lin(W.gu, a.gu);
        launch_pdl(prefill_swiglu_kernel, dim3(32, (unsigned)n), dim3(kRowThreads), 0, s, sc.y, sc.h, n, a.I,
                   pm(a.gu), a.gu.rows, pk(a.down));
        lin(W.down, a.down);
        // the residual add, then the next layer's input norm (after the last
        // layer, the final norm ahead of the LM head)
        const bool last = l + 1 == a.L;
        launch_pdl(residual_norm_kernel, dim3(n), dim3(kNormThreads), 0, s, sc.x, static_cast<const float *>(sc.y),
                   pm(a.down),
                   static_cast<const uint16_t *>(last ? a.final_norm : a.layers[l + 1].attn_norm), sc.h, n, a.H,
                   last ? pk(a.lm) : pk(a.qkv), a.eps);
    }
    return err;
}

std::string last_error(std::string err) {
    if (err.empty()) {
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) err = cudaGetErrorString(e);
    }
    return err;
}

}  // namespace

std::string prefill_tc(const PrefillTc &a, const int32_t *tokens, int T, cudaStream_t s) {
    using namespace tcdec;
    const int R = kPrefillRows;
    RowsScratch sc;
    if (!carve(a, sc)) return "prefill scratch too small";
    std::string err;
    for (int b = 0; b < a.B && err.empty(); ++b)
        for (int t0 = 0; t0 < T && err.empty(); t0 += R) {
            const int n = std::min(R, T - t0);
            launch_pdl(prefill_embed_kernel, dim3(n), dim3(kRowThreads), 0, s, tokens, (int64_t)T, b, t0,
                       static_cast<const uint16_t *>(a.embed), sc.x, a.H, a.V, a.state, 0);
            launch_pdl(prefill_rows_kernel, dim3(1), dim3(128), 0, s, sc.rows, sc.rows + R, n, b, t0,
                       static_cast<const State *>(a.state), 0, sc.skflags);
            const int chunks = std::max(1, std::min(kPrefillChunks, (t0 + n) / 128));
            err = rows_through_layers(a, sc, n, chunks, false, s);
        }
    return last_error(err);
}

std::string decode_tc(const PrefillTc &a, const int32_t *tokens, int32_t *next, float *logits, cudaStream_t s) {
    using namespace tcdec;
    const int R = kPrefillRows;
    RowsScratch sc;
    if (!carve(a, sc)) return "scratch too small";
    // the attended length is read on the device; split the positions so that
    // a long cache still spreads over the SMs, a fixed count (the isolated
    // attention's rule at max_seq) so that the same launches serve every
    // position
    const int chunks =
        std::max(1, std::min(kPrefillChunks, mk_attention_chunks(std::min(a.B, R), a.nkv, a.max_seq)));
    std::string err;
    for (int b0 = 0; b0 < a.B && err.empty(); b0 += R) {
        const int n = std::min(R, a.B - b0);
        launch_pdl(prefill_embed_kernel, dim3(n), dim3(kRowThreads), 0, s, tokens + b0, (int64_t)0, -1, 0,
                   static_cast<const uint16_t *>(a.embed), sc.x, a.H, a.V, a.state, b0);
        launch_pdl(prefill_rows_kernel, dim3(1), dim3(128), 0, s, sc.rows, sc.rows + R, n, -1, 0,
                   static_cast<const State *>(a.state), b0, sc.skflags);
        err = rows_through_layers(a, sc, n, chunks, true, s);  // ends with the final norm
        if (!err.empty()) break;
        const cudaError_t e = launch_linear_tc_packed_sk(sc.h, a.lm_w, sc.y, 2 * n, pk(a.lm), pm(a.lm), a.lm.kc,
                                                         a.lm.rows, sc.skws, sc.skflags, s, true);
        if (e != cudaSuccess) {
            err = std::string("LM head: ") + cudaGetErrorString(e);
            break;
        }
        float *pv = sc.part;  // the attention partials are free again
        int *pi = reinterpret_cast<int *>(sc.part + kPrefillRows * kArgParts);
        launch_pdl(argmax_part_kernel, dim3(kArgParts, (unsigned)n), dim3(kArgmaxThreads), 0, s,
                   static_cast<const float *>(sc.y), pm(a.lm), n, logits, a.V, b0, pv, pi);
        launch_pdl(argmax_final_kernel, dim3(n), dim3(kArgParts), 0, s, static_cast<const float *>(pv),
                   static_cast<const int *>(pi), next, b0, a.state);
    }
    if (err.empty()) launch_pdl(advance_pos_kernel, dim3(1), dim3(1), 0, s, a.state);
    return last_error(err);
}

int32_t *decode_tc_tokens(const PrefillTc &a) {
    RowsScratch sc;
    return carve(a, sc) ? sc.tok : nullptr;
}
int32_t *decode_tc_next(const PrefillTc &a) {
    RowsScratch sc;
    return carve(a, sc) ? sc.nxt : nullptr;
}

}  // namespace mk

using namespace mk;
using namespace mk::tcdec;

struct mk_tcdec {
    mk_config cfg{};
    std::string err;
    const void *embed = nullptr, *final_norm = nullptr, *lm_head = nullptr;
    std::vector<const void *> attn_norm, wq, wk, wv, wo, q_norm, k_norm, mlp_norm, wg, wu, wd;
    Layout lay{};
    uint8_t *ws = nullptr;
    uint16_t *kv = nullptr;
    int chunks = 1;                                // split-KV chunks, fixed for every position
    bool use_graph = true;
    bool warmed = false;                           // one eager step ran (kernel attributes are set)
    cudaGraphExec_t exec[2] = {nullptr, nullptr};  // the captured step without / with logits
};

static void drop_graphs(mk_tcdec *d) {
    for (auto &e : d->exec)
        if (e) {
            cudaGraphExecDestroy(e);
            e = nullptr;
        }
}

static mk_status tc_fail(mk_tcdec *d, mk_status s, const std::string &msg) {
    if (d)
        d->err = msg;
    else
        set_op_error(msg.c_str());
    return s;
}

static bool aligned16(const void *p) { return p && ((uintptr_t)p & 15u) == 0; }

extern "C" mk_status mk_tcdec_create(const mk_config *cfg, const mk_weights *w, mk_tcdec **out) {
    if (!cfg || !w || !out) return tc_fail(nullptr, MK_ERR_INVALID, "tcdec: null argument");
    *out = nullptr;
    const mk_config &c = *cfg;
    if (c.n_layers < 1 || c.hidden < 1 || c.n_heads < 1 || c.n_kv_heads < 1 || c.intermediate < 1 || c.vocab < 1 ||
        c.batch < 1 || c.max_seq < 1 || !(c.rms_eps >= 0.f) || !(c.rope_theta > 0.f))
        return tc_fail(nullptr, MK_ERR_INVALID, "tcdec: sizes must be positive");
    if (c.dtype != MK_BF16) return tc_fail(nullptr, MK_ERR_UNSUPPORTED, "tcdec: only bf16 weights");
    if (c.batch > kMaxBatch) return tc_fail(nullptr, MK_ERR_UNSUPPORTED, "tcdec: batch above 32");
    if (c.head_dim != 64 && c.head_dim != 128)
        return tc_fail(nullptr, MK_ERR_UNSUPPORTED, "tcdec: head_dim must be 64 or 128");
    if (c.n_heads % c.n_kv_heads || c.n_heads / c.n_kv_heads > 8)
        return tc_fail(nullptr, MK_ERR_UNSUPPORTED, "tcdec: n_heads must be a multiple of n_kv_heads, at most 8x");
    if (c.hidden % 64 || c.intermediate % 64 || (c.n_heads * c.head_dim) % 64)
        return tc_fail(nullptr, MK_ERR_UNSUPPORTED,
                       "tcdec: hidden, intermediate and n_heads*head_dim must be multiples of 64");
    auto d = new mk_tcdec();
    d->cfg = c;
    d->embed = w->embed;
    d->final_norm = w->final_norm;
    d->lm_head = c.tied_embeddings ? w->embed : w->lm_head;
    bool ok = aligned16(d->embed) && aligned16(d->final_norm) && aligned16(d->lm_head);
    const int L = c.n_layers;
    auto grab = [&](const void *const *src, std::vector<const void *> &dst, bool need) {
        if (!src) {
            if (need) ok = false;
            dst.assign((size_t)L, nullptr);
            return;
        }
        dst.assign(src, src + L);
        if (need)
            for (const void *p : dst) ok = ok && aligned16(p);
    };
    grab(w->attn_norm, d->attn_norm, true);
    grab(w->wq, d->wq, true);
    grab(w->wk, d->wk, true);
    grab(w->wv, d->wv, true);
    grab(w->wo, d->wo, true);
    grab(w->mlp_norm, d->mlp_norm, true);
    grab(w->wg, d->wg, true);
    grab(w->wu, d->wu, true);
    grab(w->wd, d->wd, true);
    grab(w->q_norm, d->q_norm, c.qk_norm != 0);
    grab(w->k_norm, d->k_norm, c.qk_norm != 0);
    if (!ok) {
        delete d;
        return tc_fail(nullptr, MK_ERR_INVALID, "tcdec: a weight pointer is null or not 16-byte aligned");
    }
    d->lay = layout(c);
    d->chunks = mk_attention_chunks(c.batch, c.n_kv_heads, c.max_seq);
    if (d->chunks < 1) d->chunks = 1;
    if (d->chunks > kMaxChunks) d->chunks = kMaxChunks;
    *out = d;
    return MK_OK;
}

extern "C" mk_status mk_tcdec_workspace_bytes(const mk_tcdec *d, size_t *bytes) {
    if (!d || !bytes) return MK_ERR_INVALID;
    *bytes = d->lay.total;
    return MK_OK;
}

extern "C" mk_status mk_tcdec_bind(mk_tcdec *d, void *workspace, void *kv_cache) {
    // the workspace and the cache belong to the caller; the status word is
    // cleared here (synchronously) and only ever set afterwards
    if (!d) return tc_fail(nullptr, MK_ERR_INVALID, "tcdec: null context");
    if (!workspace || ((uintptr_t)workspace & 255u) || !aligned16(kv_cache))
        return tc_fail(d, MK_ERR_INVALID, "tcdec: workspace must be 256-byte and kv_cache 16-byte aligned");
    drop_graphs(d);  // the captured steps point at the old buffers
    d->ws = static_cast<uint8_t *>(workspace);
    d->kv = static_cast<uint16_t *>(kv_cache);
    if (cudaMemset(d->ws + d->lay.status, 0, sizeof(int)) != cudaSuccess)
        return tc_fail(d, MK_ERR_CUDA, "tcdec: clearing the status word");
    return MK_OK;
}

// Queue one whole step on `s`: tokens from the workspace's token row, the
// position from its position words, the argmax (and the logits if `logits`)
// into the workspace.  Every launch reads its varying inputs from device
// memory, so the same sequence of launches, captured once, serves every step.
static mk_status enqueue_step(mk_tcdec *d, cudaStream_t s, bool logits) {
    const mk_config &c = d->cfg;
    const Layout &o = d->lay;
    void *stream = s;
    const int B = c.batch, H = c.hidden, I = c.intermediate, V = c.vocab, L = c.n_layers;
    const int nq = c.n_heads, nkv = c.n_kv_heads, hd = c.head_dim, QD = nq * hd, KD = nkv * hd;
    float *x = reinterpret_cast<float *>(d->ws + o.x);
    __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(d->ws + o.h);
    float *yq = reinterpret_cast<float *>(d->ws + o.yq), *yk = reinterpret_cast<float *>(d->ws + o.yk);
    float *yv = reinterpret_cast<float *>(d->ws + o.yv), *ya = reinterpret_cast<float *>(d->ws + o.ya);
    float *yg = reinterpret_cast<float *>(d->ws + o.yg), *yu = reinterpret_cast<float *>(d->ws + o.yu);
    float *ylm = reinterpret_cast<float *>(d->ws + o.ylm);
    float *q = reinterpret_cast<float *>(d->ws + o.q), *attn = reinterpret_cast<float *>(d->ws + o.attn);
    float *scratch = reinterpret_cast<float *>(d->ws + o.scratch);
    int *status = reinterpret_cast<int *>(d->ws + o.status);
    const int32_t *tok = reinterpret_cast<const int32_t *>(d->ws + o.tok);
    int32_t *nxt = reinterpret_cast<int32_t *>(d->ws + o.nxt);
    const int *posw = reinterpret_cast<const int *>(d->ws + o.posw);
    const size_t layer_elems = (size_t)B * nkv * c.max_seq * hd;
    mk_status st = MK_OK;
    auto lin = [&](const void *xin, const void *wt, float *y, int K, int M) {
        if (st == MK_OK && mk_linear_tc(xin, wt, y, 2 * B, K, M, stream) != MK_OK) {
            st = MK_ERR_CUDA;
            d->err = std::string("tcdec: ") + op_error();
        }
    };
    const dim3 rows_grid(8, (unsigned)B);
    embed_kernel<<<B, kRowThreads, 0, s>>>(tok, static_cast<const uint16_t *>(d->embed), x, H, V, status);
    for (int l = 0; l < L && st == MK_OK; ++l) {
        uint16_t *kc = d->kv + (size_t)l * layer_elems, *vc = d->kv + (size_t)(L + l) * layer_elems;
        norm_hilo_kernel<<<B, kRowThreads, 0, s>>>(x, static_cast<const uint16_t *>(d->attn_norm[l]), h, B, H,
                                                   c.rms_eps);
        lin(h, d->wq[l], yq, H, QD);
        lin(h, d->wk[l], yk, H, KD);
        lin(h, d->wv[l], yv, H, KD);
        if (st != MK_OK) break;
        qkv_post_kernel<<<dim3((unsigned)(nq + 2 * nkv), (unsigned)B), hd, (hd + 32) * sizeof(float), s>>>(
            yq, yk, yv, B, nq, nkv, hd, static_cast<const uint16_t *>(d->q_norm[l]),
            static_cast<const uint16_t *>(d->k_norm[l]), c.qk_norm, c.rms_eps, (double)c.rope_theta, posw, q, kc, vc,
            c.max_seq);
        const cudaError_t ea =
            launch_attention_dev(q, kc, vc, B, nq, nkv, hd, c.max_seq, posw + 1, d->chunks, attn, scratch, s);
        if (ea != cudaSuccess) {
            st = MK_ERR_CUDA;
            d->err = std::string("tcdec: attention: ") + cudaGetErrorString(ea);
            break;
        }
        cast_hilo_kernel<<<rows_grid, kRowThreads, 0, s>>>(attn, h, B, QD);
        lin(h, d->wo[l], ya, QD, H);
        residual_add_kernel<<<rows_grid, kRowThreads, 0, s>>>(x, ya, B, H);
        norm_hilo_kernel<<<B, kRowThreads, 0, s>>>(x, static_cast<const uint16_t *>(d->mlp_norm[l]), h, B, H,
                                                   c.rms_eps);
        lin(h, d->wg[l], yg, H, I);
        lin(h, d->wu[l], yu, H, I);
        swiglu_hilo_kernel<<<dim3(32, (unsigned)B), kRowThreads, 0, s>>>(yg, yu, h, B, I);
        lin(h, d->wd[l], ya, I, H);
        residual_add_kernel<<<rows_grid, kRowThreads, 0, s>>>(x, ya, B, H);
    }
    if (st != MK_OK) return st;
    norm_hilo_kernel<<<B, kRowThreads, 0, s>>>(x, static_cast<const uint16_t *>(d->final_norm), h, B, H, c.rms_eps);
    lin(h, d->lm_head, ylm, H, V);
    if (st != MK_OK) return st;
    lm_argmax_kernel<<<B, kArgmaxThreads, 0, s>>>(ylm, logits ? reinterpret_cast<float *>(d->ws + o.lg) : nullptr,
                                                  nxt, B, V, status);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return tc_fail(d, MK_ERR_CUDA, std::string("tcdec: ") + cudaGetErrorString(e));
    return MK_OK;
}

// Capture enqueue_step once (per logits / no-logits) into an executable graph.
static mk_status capture_step(mk_tcdec *d, bool logits) {
    cudaStream_t cap;
    cudaError_t e = cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking);
    if (e != cudaSuccess) return tc_fail(d, MK_ERR_CUDA, std::string("tcdec: ") + cudaGetErrorString(e));
    e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeRelaxed);
    if (e != cudaSuccess) {
        cudaStreamDestroy(cap);
        return tc_fail(d, MK_ERR_CUDA, std::string("tcdec: begin capture: ") + cudaGetErrorString(e));
    }
    const mk_status st = enqueue_step(d, cap, logits);
    cudaGraph_t g = nullptr;
    e = cudaStreamEndCapture(cap, &g);
    cudaStreamDestroy(cap);
    if (st != MK_OK || e != cudaSuccess) {
        if (g) cudaGraphDestroy(g);
        return st != MK_OK ? st : tc_fail(d, MK_ERR_CUDA, std::string("tcdec: end capture: ") + cudaGetErrorString(e));
    }
    e = cudaGraphInstantiate(&d->exec[logits ? 1 : 0], g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return tc_fail(d, MK_ERR_CUDA, std::string("tcdec: instantiate: ") + cudaGetErrorString(e));
    return MK_OK;
}

extern "C" mk_status mk_tcdec_step(mk_tcdec *d, const int32_t *d_tokens, int pos, int32_t *d_next, float *d_logits,
                                   void *stream) {
    if (!d) return tc_fail(nullptr, MK_ERR_INVALID, "tcdec: null context");
    if (!d->ws) return tc_fail(d, MK_ERR_STATE, "tcdec: mk_tcdec_step before mk_tcdec_bind");
    const mk_config &c = d->cfg;
    if (!d_tokens || !d_next) return tc_fail(d, MK_ERR_INVALID, "tcdec: null token buffer");
    if (pos < 0 || pos >= c.max_seq) return tc_fail(d, MK_ERR_INVALID, "tcdec: position outside the cache");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Layout &o = d->lay;
    const int B = c.batch;
    const bool logits = d_logits != nullptr;
    cudaError_t e = cudaMemcpyAsync(d->ws + o.tok, d_tokens, (size_t)B * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return tc_fail(d, MK_ERR_CUDA, std::string("tcdec: tokens: ") + cudaGetErrorString(e));
    set_pos_kernel<<<1, 1, 0, s>>>(reinterpret_cast<int *>(d->ws + o.posw), pos);
    mk_status st;
    if (d->use_graph && d->warmed) {
        if (!d->exec[logits ? 1 : 0]) {
            st = capture_step(d, logits);
            if (st != MK_OK) return st;
        }
        e = cudaGraphLaunch(d->exec[logits ? 1 : 0], s);
        if (e != cudaSuccess) return tc_fail(d, MK_ERR_CUDA, std::string("tcdec: graph launch: ") + cudaGetErrorString(e));
    } else {
        st = enqueue_step(d, s, logits);  // the first step runs eagerly: it sets the kernels' attributes
        if (st != MK_OK) return st;
        d->warmed = true;
    }
    e = cudaMemcpyAsync(d_next, d->ws + o.nxt, (size_t)B * 4, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && logits)
        e = cudaMemcpyAsync(d_logits, d->ws + o.lg, (size_t)B * c.vocab * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return tc_fail(d, MK_ERR_CUDA, std::string("tcdec: outputs: ") + cudaGetErrorString(e));
    return MK_OK;
}

extern "C" mk_status mk_tcdec_status(mk_tcdec *d, int *status, void *stream) {
    if (!d || !status) return MK_ERR_INVALID;
    if (!d->ws) return tc_fail(d, MK_ERR_STATE, "tcdec: not bound");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(status, d->ws + d->lay.status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return tc_fail(d, MK_ERR_CUDA, "tcdec: reading the status word");
    return MK_OK;
}

extern "C" const char *mk_tcdec_last_error(const mk_tcdec *d) { return d ? d->err.c_str() : op_error(); }

extern "C" mk_status mk_tcdec_destroy(mk_tcdec *d) {
    if (d) drop_graphs(d);
    delete d;
    return MK_OK;
}

extern "C" mk_status mk_tcdec_set_graph(mk_tcdec *d, int on) {
    if (!d) return tc_fail(nullptr, MK_ERR_INVALID, "tcdec: null context");
    d->use_graph = on != 0;
    if (!d->use_graph) drop_graphs(d);
    return MK_OK;
}
