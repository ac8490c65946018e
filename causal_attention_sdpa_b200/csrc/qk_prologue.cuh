// QK-Norm + rotary prologue of q and k, and its gradient: the step before attention in the
// modded-nanogpt README's "modernised architecture" item (rotary embeddings, QK-Norm).  For each
// row x (D values) of head bh at token t:
//   n = x / max(|x|, 1e-12)                                    (QK-Norm, no gain)
//   y[i] = n[i] cos a_i - n[i + D/2] sin a_i,  y[i + D/2] = n[i] sin a_i + n[i + D/2] cos a_i,
//   a_i = t * base^(-2i/D)                                     (rotary, half-split pairs)
// Gradient: dn = R^T dy (rotate back), dx = (dn - n (n . dn)) / |x| (dn / 1e-12 below the clamp).
//
// Memory-bound (one read and one write of q and k per pass), so the kernels run on the CUDA
// cores with 16-byte accesses: a row is served by G = D/16 consecutive lanes, lane j of the group
// holding the 8 elements [8j, 8j + 8) of the first half and the 8 elements [D/2 + 8j, D/2 + 8j + 8)
// of the second, i.e. both members of its 8 rotation pairs; only the norm needs a reduction over
// the group.  The grid is persistent (a few blocks per SM, grid-stride over rows) so a lane's 8
// rotation frequencies are computed once.  The angle is reduced to one revolution in fp64
// (t * base^(-2i/D) / 2 pi, minus its nearest integer), so the hardware sine and cosine only ever
// see |a| <= pi, where their absolute error is about 1e-6; an fp32 product t * base^(-2i/D) would
// already be off by up to 5e-4 rad at t = 8192.  Rows are addressed through [b, h, t, d] strides,
// so the inputs may be the q and k columns of a fused [B, T, 3, H, D] projection and the outputs
// any layout the attention kernels accept.
#pragma once

#include "attn_fwd.cuh"

namespace gpt_attn {

struct PrologueParams {
    const __nv_bfloat16* x[2];     // raw q, k
    const __nv_bfloat16* dy[2];    // backward: gradients of the prologue outputs
    __nv_bfloat16* out[2];         // forward: y; backward: dx
    Strides xs[2], dys[2], outs[2];
    int H, T;
    long long rows;                // B * H * T per tensor
    int norm;                      // 1: QK-Norm
    float base;                    // rope base; <= 1: no rotation
    int token_major;               // 1: rows in (b, t, h) order, else (b, h, t)
};

// Head and token of linear row `row`.  Rows are walked in the order of the input's memory: for
// q and k read out of a fused [B, T, 3, H, D] projection the heads of one token are adjacent
// ((b, t, h) order), for a [B, H, T, D] tensor the tokens of one head ((b, h, t) order), so the
// rows that all blocks handle at one time cover a dense stretch of memory.
__device__ __forceinline__ void prologue_row(const PrologueParams& p, long long row, int& bh, int& t) {
    if (p.token_major) {
        const long long bt = row / p.H;              // b * T + t
        const int h = (int)(row - bt * p.H);
        const int b = (int)(bt / p.T);
        t = (int)(bt - (long long)b * p.T);
        bh = b * p.H + h;
    } else {
        bh = (int)(row / p.T);
        t = (int)(row - (long long)bh * p.T);
    }
}

constexpr int kPrologueThreads = 256;

__device__ __forceinline__ void unpack_bf16x8(const uint4 u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* p, float (&f)[8]) {
    unpack_bf16x8(*reinterpret_cast<const uint4*>(p), f);
}

__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* p, const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
        w[e] = *reinterpret_cast<const uint32_t*>(&t);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Revolutions per token of every pair i < D/2, base^(-2i/D) / (2 pi), in fp64, into shared memory
// (computed once per block of the persistent grid).
template <int D>
__device__ __forceinline__ void prologue_rev_per_token(float base, double* rev) {
    if (threadIdx.x < D / 2) {
        const double lb = base > 1.f ? log2((double)base) : 0.0;
        rev[threadIdx.x] = base > 1.f ? exp2(-2.0 * (double)threadIdx.x / (double)D * lb) * 0.15915494309189535 : 0.0;
    }
    __syncthreads();
}

// cos and sin of t * 2 pi * rev, the angle first reduced to [-pi, pi] in fp64.
__device__ __forceinline__ void prologue_angle(int t, double rev, float& c, float& s) {
    const double r = (double)t * rev;
    const float a = (float)(r - rint(r)) * 6.283185307179586f;
    __sincosf(a, &s, &c);
}

// The same for the angles of pairs 8j .. 8j + 7 at token t (rev points at pair 8j).
__device__ __forceinline__ void prologue_angles(int t, const double* rev, float (&c)[8], float (&s)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) prologue_angle(t, rev[e], c[e], s[e]);
}

// Sum over the G lanes of a row's group (G a power of two, groups aligned within the warp).
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int off = G / 2; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 4)
qk_prologue_fwd_kernel(const PrologueParams p) {
    constexpr int G = D / 16, H2 = D / 2, kRows = kPrologueThreads / G;
    constexpr int U = 2;                             // rows per lane group and iteration
    const int which = blockIdx.y;                    // 0: q, 1: k
    const int j = threadIdx.x % G;
    __shared__ double rev[D / 2];
    prologue_rev_per_token<D>(p.base, rev);
    const __nv_bfloat16* xb = p.x[which];
    __nv_bfloat16* yb = p.out[which];
    const Strides xs = p.xs[which], ys = p.outs[which];
    const long long stride = (long long)gridDim.x * kRows;
    // Each iteration takes U rows a grid stride apart, all loads issued before any arithmetic, so
    // 4 x 16 bytes per lane are in flight.  The loop bound is taken on the warp's first row, so
    // every lane of a warp runs the same iterations and takes part in every shuffle; lanes whose
    // row is past the end compute on zeros and store nothing.
    for (long long row0 = (long long)blockIdx.x * kRows + (threadIdx.x & ~31) / G; row0 < p.rows;
         row0 += U * stride) {
        bool valid[U];
        int bh[U], t[U];
        uint4 ra[U], rb[U];                          // elements 8j + e and D/2 + 8j + e, still bf16
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long row = row0 + u * stride + (threadIdx.x & 31) / G;
            valid[u] = row < p.rows;
            bh[u] = 0, t[u] = 0;
            if (valid[u]) prologue_row(p, row, bh[u], t[u]);
            ra[u] = rb[u] = make_uint4(0u, 0u, 0u, 0u);
            if (valid[u]) {
                const __nv_bfloat16* x = xb + xs.row(bh[u], p.H, t[u]) + 8 * j;
                ra[u] = *reinterpret_cast<const uint4*>(x);
                rb[u] = *reinterpret_cast<const uint4*>(x + H2);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float a[8], b[8];
            unpack_bf16x8(ra[u], a);
            unpack_bf16x8(rb[u], b);
            float inv = 1.f;
            if (p.norm) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(a[e], a[e], fmaf(b[e], b[e], ss));
                inv = 1.f / fmaxf(sqrtf(group_sum<G>(ss)), 1e-12f);
            }
            // rotate pair by pair, packing the outputs as they are produced
            uint32_t oa[4], ob[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                float c0, s0, c1, s1;
                prologue_angle(t[u], rev[8 * j + e], c0, s0);
                prologue_angle(t[u], rev[8 * j + e + 1], c1, s1);
                const float u0 = a[e] * inv, w0 = b[e] * inv, u1 = a[e + 1] * inv, w1 = b[e + 1] * inv;
                oa[e >> 1] = pack_bf16x2(u0 * c0 - w0 * s0, u1 * c1 - w1 * s1);
                ob[e >> 1] = pack_bf16x2(u0 * s0 + w0 * c0, u1 * s1 + w1 * c1);
            }
            if (valid[u]) {
                __nv_bfloat16* y = yb + ys.row(bh[u], p.H, t[u]) + 8 * j;
                *reinterpret_cast<uint4*>(y) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
                *reinterpret_cast<uint4*>(y + H2) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 4)
qk_prologue_bwd_kernel(const PrologueParams p) {
    constexpr int G = D / 16, H2 = D / 2, kRows = kPrologueThreads / G;
    const int which = blockIdx.y;
    const int j = threadIdx.x % G;
    __shared__ double rev[D / 2];
    prologue_rev_per_token<D>(p.base, rev);
    const __nv_bfloat16* xb = p.x[which];
    const __nv_bfloat16* gb = p.dy[which];
    __nv_bfloat16* db = p.out[which];
    const Strides xs = p.xs[which], gs = p.dys[which], ds = p.outs[which];
    for (long long row0 = (long long)blockIdx.x * kRows + (threadIdx.x & ~31) / G; row0 < p.rows;
         row0 += (long long)gridDim.x * kRows) {    // warp-uniform bound, as in the forward kernel
        const long long row = row0 + (threadIdx.x & 31) / G;
        const bool valid = row < p.rows;
        int bh = 0, t = 0;
        if (valid) prologue_row(p, row, bh, t);
        const __nv_bfloat16* x = xb + xs.row(bh, p.H, t) + 8 * j;
        const __nv_bfloat16* g = gb + gs.row(bh, p.H, t) + 8 * j;
        float ga[8] = {}, gb2[8] = {}, xa[8] = {}, xb2[8] = {};
        if (valid) {
            load_bf16x8(g, ga);
            load_bf16x8(g + H2, gb2);
            if (p.norm) {
                load_bf16x8(x, xa);
                load_bf16x8(x + H2, xb2);
            }
        }
        float c[8], s[8], da[8], db2[8];
        prologue_angles(t, rev + 8 * j, c, s);
#pragma unroll
        for (int e = 0; e < 8; ++e) {                // rotate back: dn = R^T dy
            da[e] = ga[e] * c[e] + gb2[e] * s[e];
            db2[e] = -ga[e] * s[e] + gb2[e] * c[e];
        }
        if (p.norm) {
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = fmaf(xa[e], xa[e], fmaf(xb2[e], xb2[e], ss));
            const float r = sqrtf(group_sum<G>(ss));
            const float inv = r > 1e-12f ? 1.f / r : 0.f;
            float nd = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) nd = fmaf(xa[e], da[e], fmaf(xb2[e], db2[e], nd));
            nd = group_sum<G>(nd) * inv;             // n . dn; every lane of the warp shuffles
            if (r > 1e-12f) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    da[e] = (da[e] - xa[e] * inv * nd) * inv;
                    db2[e] = (db2[e] - xb2[e] * inv * nd) * inv;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    da[e] *= 1e12f;
                    db2[e] *= 1e12f;
                }
            }
        }
        if (valid) {
            __nv_bfloat16* d = db + ds.row(bh, p.H, t) + 8 * j;
            store_bf16x8(d, da);
            store_bf16x8(d + H2, db2);
        }
    }
}

// Token-major inputs (the q and k of a fused [B, T, 3, H, D] projection): the H heads of a token
// are adjacent in memory and share their rotation angles, so a lane group takes a whole token, works
// out its 8 angles once, and runs the token's heads two at a time, both heads' loads issued before
// any arithmetic.  Same results as the kernels above (the same operations on each row).
template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 4)
qk_prologue_fwd_tok_kernel(const PrologueParams p) {
    constexpr int G = D / 16, H2 = D / 2, kGroups = kPrologueThreads / G;
    constexpr int UH = 1;                            // heads per batch of loads
    const int which = blockIdx.y;
    const int j = threadIdx.x % G;
    __shared__ double rev[D / 2];
    prologue_rev_per_token<D>(p.base, rev);
    const __nv_bfloat16* xb = p.x[which];
    __nv_bfloat16* yb = p.out[which];
    const Strides xs = p.xs[which], ys = p.outs[which];
    const long long n_tok = p.rows / p.H;            // B * T
    // warp-uniform loop bound (the warp's first token), as in the row kernels
    for (long long tok0 = (long long)blockIdx.x * kGroups + (threadIdx.x & ~31) / G; tok0 < n_tok;
         tok0 += (long long)gridDim.x * kGroups) {
        const long long tok = tok0 + (threadIdx.x & 31) / G;
        const bool valid = tok < n_tok;
        const int b = valid ? (int)(tok / p.T) : 0;
        const int t = valid ? (int)(tok - (long long)b * p.T) : 0;
        float c[8], s[8];
        prologue_angles(t, rev + 8 * j, c, s);
        // the token's head 0; head h sits h head strides further
        const __nv_bfloat16* xt = xb + (long long)b * xs.b + (long long)t * xs.t + 8 * j;
        __nv_bfloat16* yt = yb + (long long)b * ys.b + (long long)t * ys.t + 8 * j;
        for (int h0 = 0; h0 < p.H; h0 += UH) {
            uint4 ra[UH], rb[UH];
#pragma unroll
            for (int u = 0; u < UH; ++u) {
                ra[u] = rb[u] = make_uint4(0u, 0u, 0u, 0u);
                if (valid && h0 + u < p.H) {
                    const __nv_bfloat16* x = xt + (long long)(h0 + u) * xs.h;
                    ra[u] = *reinterpret_cast<const uint4*>(x);
                    rb[u] = *reinterpret_cast<const uint4*>(x + H2);
                }
            }
#pragma unroll
            for (int u = 0; u < UH; ++u) {
                float a[8], bb[8];
                unpack_bf16x8(ra[u], a);
                unpack_bf16x8(rb[u], bb);
                float inv = 1.f;
                if (p.norm) {
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(a[e], a[e], fmaf(bb[e], bb[e], ss));
                    inv = 1.f / fmaxf(sqrtf(group_sum<G>(ss)), 1e-12f);
                }
                uint32_t oa[4], ob[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float u0 = a[e] * inv, w0 = bb[e] * inv, u1 = a[e + 1] * inv, w1 = bb[e + 1] * inv;
                    oa[e >> 1] = pack_bf16x2(u0 * c[e] - w0 * s[e], u1 * c[e + 1] - w1 * s[e + 1]);
                    ob[e >> 1] = pack_bf16x2(u0 * s[e] + w0 * c[e], u1 * s[e + 1] + w1 * c[e + 1]);
                }
                if (valid && h0 + u < p.H) {
                    __nv_bfloat16* y = yt + (long long)(h0 + u) * ys.h;
                    *reinterpret_cast<uint4*>(y) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
                    *reinterpret_cast<uint4*>(y + H2) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
                }
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kPrologueThreads, 4)
qk_prologue_bwd_tok_kernel(const PrologueParams p) {
    constexpr int G = D / 16, H2 = D / 2, kGroups = kPrologueThreads / G;
    const int which = blockIdx.y;
    const int j = threadIdx.x % G;
    __shared__ double rev[D / 2];
    prologue_rev_per_token<D>(p.base, rev);
    const __nv_bfloat16* xb = p.x[which];
    const __nv_bfloat16* gb = p.dy[which];
    __nv_bfloat16* db = p.out[which];
    const Strides xs = p.xs[which], gs = p.dys[which], ds = p.outs[which];
    const long long n_tok = p.rows / p.H;
    for (long long tok0 = (long long)blockIdx.x * kGroups + (threadIdx.x & ~31) / G; tok0 < n_tok;
         tok0 += (long long)gridDim.x * kGroups) {
        const long long tok = tok0 + (threadIdx.x & 31) / G;
        const bool valid = tok < n_tok;
        const int b = valid ? (int)(tok / p.T) : 0;
        const int t = valid ? (int)(tok - (long long)b * p.T) : 0;
        float c[8], s[8];
        prologue_angles(t, rev + 8 * j, c, s);
        const __nv_bfloat16* gt = gb + (long long)b * gs.b + (long long)t * gs.t + 8 * j;
        const __nv_bfloat16* xt = xb + (long long)b * xs.b + (long long)t * xs.t + 8 * j;
        __nv_bfloat16* dt = db + (long long)b * ds.b + (long long)t * ds.t + 8 * j;
        for (int h = 0; h < p.H; ++h) {
            float ga[8] = {}, gb2[8] = {}, xa[8] = {}, xb2[8] = {};
            if (valid) {
                const __nv_bfloat16* g = gt + (long long)h * gs.h;
                load_bf16x8(g, ga);
                load_bf16x8(g + H2, gb2);
                if (p.norm) {
                    const __nv_bfloat16* x = xt + (long long)h * xs.h;
                    load_bf16x8(x, xa);
                    load_bf16x8(x + H2, xb2);
                }
            }
            float da[8], db2[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {            // rotate back: dn = R^T dy
                da[e] = ga[e] * c[e] + gb2[e] * s[e];
                db2[e] = -ga[e] * s[e] + gb2[e] * c[e];
            }
            if (p.norm) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(xa[e], xa[e], fmaf(xb2[e], xb2[e], ss));
                const float r = sqrtf(group_sum<G>(ss));
                const float inv = r > 1e-12f ? 1.f / r : 0.f;
                float nd = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) nd = fmaf(xa[e], da[e], fmaf(xb2[e], db2[e], nd));
                nd = group_sum<G>(nd) * inv;
                if (r > 1e-12f) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        da[e] = (da[e] - xa[e] * inv * nd) * inv;
                        db2[e] = (db2[e] - xb2[e] * inv * nd) * inv;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        da[e] *= 1e12f;
                        db2[e] *= 1e12f;
                    }
                }
            }
            if (valid) {
                __nv_bfloat16* d = dt + (long long)h * ds.h;
                store_bf16x8(d, da);
                store_bf16x8(d + H2, db2);
            }
        }
    }
}

}  // namespace gpt_attn
