// Decode attention: one new query per (batch, head) against its cached keys and values, the
// inner step of the generation loop of "Un GPT desde cero + nanoGPT" (Laboratorio L2.1,
// generate), which runs the model on the growing sequence and keeps the last position.  The
// query is the last token of a sequence of L tokens: it sees keys [lo, L), lo = max(0, L - W)
// with a window W >= 1, else 0.
//
// Per query this is a matrix-vector product over the cached keys and another over the values:
// about one flop per byte read, so the kernel is bound by HBM bandwidth and runs on the CUDA
// cores (no tensor-core tile would be more than 1/128 full).  Keys are split into chunks so
// that even a single sequence spreads over many SMs (split-K):
//   attn_decode_split_kernel   grid (B*H, n_split), 128 threads.  Scores of the chunk with
//                              D/8 threads per key row (16-byte loads, a warp reads 4 whole
//                              rows), softmax pieces relative to the chunk max, then
//                              sum_j p_j V_j with D/8 threads per value row.  With one split it
//                              writes O and lse; otherwise an fp32 partial (m, l, o) per split.
//   attn_decode_combine_kernel grid B*H, D threads: rescales the partials to their common max,
//                              O = sum o_s / sum l_s, lse = M + log l (natural log).
#pragma once

#include "sm100.cuh"

namespace gpt_attn {

constexpr int kDecodeThreads = 128;
constexpr int kDecodeMaxChunk = 4096;       // keys per split (scores kept in shared memory)

struct DecodeParams {
    const __nv_bfloat16* q;     // [BH, D]
    const __nv_bfloat16* k;     // [BH, T_max, D]
    const __nv_bfloat16* v;     // [BH, T_max, D]
    const int* lens;            // [B] tokens per sequence (device), clamped to [0, T_max]
    __nv_bfloat16* o;           // [BH, D]
    float* lse;                 // [BH]
    float* part_o;              // [BH, n_split, D]   unnormalised, relative to the split's max
    float* part_ml;             // [BH, n_split, 2]   (max, sum), log2 units
    int H;
    int T_max;
    int n_split;
    int chunk;                  // keys per split
    int window;                 // <= 0: no window
    float scale_log2;           // scale * log2(e)
};

__device__ __forceinline__ void decode_range(const DecodeParams& p, int bh, int& lo, int& L) {
    L = __ldg(p.lens + bh / p.H);
    L = L < 0 ? 0 : (L > p.T_max ? p.T_max : L);
    lo = (p.window > 0 && L - p.window > 0) ? L - p.window : 0;
}

constexpr int kDecodeBlocksPerSm = 6;     // resident split CTAs per SM (registers capped to fit)

template <int D>
__global__ void __launch_bounds__(kDecodeThreads, kDecodeBlocksPerSm)
attn_decode_split_kernel(const DecodeParams p) {
    constexpr int G = D / 8;                          // threads per row, 8 elements (16 bytes) each
    constexpr int R = kDecodeThreads / G;             // rows handled at once
    extern __shared__ float dsm[];                    // max(chunk, R * D) floats: chunk scores /
                                                      // probabilities, then R x D partial sums
    __shared__ float red[kDecodeThreads / 32];
    const int bh = blockIdx.x, s = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    int lo, L;
    decode_range(p, bh, lo, L);
    const int j0 = lo + s * p.chunk;
    const int j1 = min(L, j0 + p.chunk);
    const int n = j1 - j0;                            // keys of this split (may be <= 0)
    const int g = tid % G, r = tid / G;

    // q slice of this thread, scaled to log2 units
    float qv[8];
    {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.q + (size_t)bh * D) + g);
        const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
            qv[2 * e] = f.x * p.scale_log2;
            qv[2 * e + 1] = f.y * p.scale_log2;
        }
    }
    const __nv_bfloat16* kh = p.k + (size_t)bh * p.T_max * D;
    const __nv_bfloat16* vh = p.v + (size_t)bh * p.T_max * D;

    // scores: G threads per key row, reduced across the group with shuffles.  Each thread keeps
    // kU rows in flight (HBM latency is hidden by loads in flight, not by threads alone).  Every
    // thread runs the same number of iterations (rows past the chunk are predicated off), so the
    // whole warp takes part in every shuffle.
    constexpr int kU = 12;
    float mloc = -INFINITY;
    for (int base = 0; base < n; base += kU * R) {
        uint4 raw[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int jj = base + u * R + r;
            raw[u] = jj < n ? __ldg(reinterpret_cast<const uint4*>(kh + (size_t)(j0 + jj) * D) + g)
                            : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const uint32_t w4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                acc = fmaf(qv[2 * e], f.x, acc);
                acc = fmaf(qv[2 * e + 1], f.y, acc);
            }
#pragma unroll
            for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            const int jj = base + u * R + r;
            if (jj < n) {
                if (g == 0) dsm[jj] = acc;
                mloc = fmaxf(mloc, acc);
            }
        }
    }
    // chunk max over the block
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, off));
    if (lane == 0) red[wid] = mloc;
    __syncthreads();
    float m = red[0];
#pragma unroll
    for (int w = 1; w < kDecodeThreads / 32; ++w) m = fmaxf(m, red[w]);
    __syncthreads();
    // probabilities relative to the chunk max, and their sum
    float lsum = 0.f;
    for (int jj = tid; jj < n; jj += kDecodeThreads) {
        const float pj = exp2f(dsm[jj] - m);
        dsm[jj] = pj;
        lsum += pj;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    if (lane == 0) red[wid] = lsum;
    __syncthreads();
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeThreads / 32; ++w) l += red[w];
    // o = sum_j p_j V_j: G threads per value row, R rows at once (kV of them in flight per
    // thread), then a sum over the R groups
    constexpr int kV = 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int base = 0; base < n; base += kV * R) {
        uint4 raw[kV];
        float pj[kV];
#pragma unroll
        for (int u = 0; u < kV; ++u) {
            const int jj = base + u * R + r;
            const bool valid = jj < n;
            raw[u] = valid ? __ldg(reinterpret_cast<const uint4*>(vh + (size_t)(j0 + jj) * D) + g)
                           : make_uint4(0u, 0u, 0u, 0u);
            pj[u] = valid ? dsm[jj] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kV; ++u) {
            const uint32_t w4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                acc[2 * e] = fmaf(pj[u], f.x, acc[2 * e]);
                acc[2 * e + 1] = fmaf(pj[u], f.y, acc[2 * e + 1]);
            }
        }
    }
    __syncthreads();                                   // the chunk's probabilities are no longer read
    float* part = dsm;                                 // [R][D]
#pragma unroll
    for (int e = 0; e < 8; ++e) part[r * D + g * 8 + e] = acc[e];
    __syncthreads();
    if (tid < D) {
        float od = 0.f;
#pragma unroll
        for (int rr = 0; rr < R; ++rr) od += part[rr * D + tid];
        if (p.n_split == 1) {
            const bool any = n > 0;
            p.o[(size_t)bh * D + tid] = __float2bfloat16_rn(any ? od / l : 0.f);
            if (tid == 0) p.lse[bh] = any ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        } else {
            const size_t ps = (size_t)bh * p.n_split + s;
            p.part_o[ps * D + tid] = od;
            if (tid == 0) {
                p.part_ml[2 * ps] = n > 0 ? m : -INFINITY;
                p.part_ml[2 * ps + 1] = n > 0 ? l : 0.f;
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(D)
attn_decode_combine_kernel(const DecodeParams p) {
    const int bh = blockIdx.x, d = threadIdx.x;
    const float* ml = p.part_ml + (size_t)bh * p.n_split * 2;
    float M = -INFINITY;
    for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, ml[2 * s]);
    float l = 0.f, od = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < p.n_split; ++s) {
            const float w = exp2f(ml[2 * s] - M);     // 0 for empty splits (max -inf)
            l += w * ml[2 * s + 1];
            od += w * p.part_o[((size_t)bh * p.n_split + s) * D + d];
        }
    }
    const bool any = l > 0.f;
    p.o[(size_t)bh * D + d] = __float2bfloat16_rn(any ? od / l : 0.f);
    if (d == 0) p.lse[bh] = any ? (M + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace gpt_attn
