// backward.cuh -- gradients of exact attention with respect to q, k and v.
//
// The method (scirs2-neural 0.4.3, src/layers/flash_attention.rs, flash_backward_head: FA-2's
// backward, Algorithm 4 of Dao 2023): with the row logsumexp saved by the forward, the
// probabilities are recomputed tile by tile instead of stored,
//   P_ij = exp(scale * q_i . k_j [+ mask_ij] - lse_i) (0 for masked keys and rows without keys)
//   D_i  = sum_d dO_id O_id
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dV_j += P_ij dO_i,   dK_j += scale dS_ij q_i,   dQ_i += scale dS_ij k_j
// Grouped-query heads (scirs2-neural 0.4.4 grouped_query_attention.rs, backward): a kv head's
// dK and dV are summed over the q heads of its group.  With RoPE the scores use the rotated q
// and k, and the gradients are rotated back (the transpose of a rotation is the rotation by the
// negated angle).
//
// This file is the fp32 path (ATTN_FP32 inputs, CUDA cores); bf16 inputs take the tensor-core
// kernels of backward_mma.cuh.  Layout of the work:
//   bwd_prep_q_kernel    one warp per (b, i, h): D_i, dO and q (rotated) as fp32 copies
//   bwd_prep_kv_kernel   one warp per (b, j, kvh): k (rotated) and v as fp32 copies
//   bwd_dq_kernel<D>     one CTA per (b, h, 64 query rows), 4 threads per row, each owning D/4
//                        contiguous dims; K/V tiles of 64 keys staged in shared memory
//   bwd_dkdv_kernel<D>   one CTA per (b, kv head, 64 keys), 4 threads per key; Q/dO tiles of 64
//                        rows of every q head of the group staged in shared memory, so the
//                        group sum needs no atomics
// Both main kernels recompute S (the method's recomputation) and make each product a
// four-thread shuffle reduction; they never write partial results to memory.
#pragma once

#include "common.cuh"

namespace attn {

constexpr int kBwdRows = 64;        // query rows (dq kernel) or keys (dk/dv kernel) per CTA
constexpr int kBwdTile = 64;        // keys (dq) or query rows (dk/dv) staged per step
constexpr int kBwdThreads = 256;    // 4 threads per row

template <typename T>
__device__ __forceinline__ float load_as_f32(const T* p) {
    if constexpr (sizeof(T) == 2) return __bfloat162float(*p);
    else return *p;
}

// Rotate the pair (x0, x1) by +theta (sgn = +1) or -theta (sgn = -1) with cs = (cos, sin).
__device__ __forceinline__ void rot_pair(float& x0, float& x1, float2 cs, float sgn) {
    const float s = sgn * cs.y;
    const float y0 = x0 * cs.x - x1 * s;
    const float y1 = x0 * s + x1 * cs.x;
    x0 = y0;
    x1 = y1;
}

// One warp per (b, i, h) row: Dvec = dO . O, dOf = dO, Qf = q rotated at q_pos0 + i.
template <typename T>
__global__ void bwd_prep_q_kernel(const T* __restrict__ q, const T* __restrict__ o, const T* __restrict__ dout,
                                  float* __restrict__ Qf, float* __restrict__ dOf, float* __restrict__ Dvec,
                                  const float2* __restrict__ tab, long nrows, int Sq, int Hq, int D, int q_pos0) {
    const int lane = threadIdx.x & 31;
    const long row = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (row >= nrows) return;
    const int h = static_cast<int>(row % Hq);
    const int i = static_cast<int>((row / Hq) % Sq);
    const long b = row / (static_cast<long>(Hq) * Sq);
    const long off = row * D;
    float acc = 0.f;
    for (int d = 2 * lane; d < D; d += 64) {
        const float g0 = load_as_f32(dout + off + d), g1 = load_as_f32(dout + off + d + 1);
        acc = fmaf(g0, load_as_f32(o + off + d), acc);
        acc = fmaf(g1, load_as_f32(o + off + d + 1), acc);
        dOf[off + d] = g0;
        dOf[off + d + 1] = g1;
        float x0 = load_as_f32(q + off + d), x1 = load_as_f32(q + off + d + 1);
        if (tab != nullptr) rot_pair(x0, x1, tab[static_cast<long>(q_pos0 + i) * (D / 2) + d / 2], 1.f);
        Qf[off + d] = x0;
        Qf[off + d + 1] = x1;
    }
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
    if (lane == 0) Dvec[(b * Hq + h) * Sq + i] = acc;
}

// One warp per (b, j, kvh) row: Kf = k rotated at j, Vf = v.
template <typename T>
__global__ void bwd_prep_kv_kernel(const T* __restrict__ k, const T* __restrict__ v, float* __restrict__ Kf,
                                   float* __restrict__ Vf, const float2* __restrict__ tab, long nrows, int Skv,
                                   int Hkv, int D) {
    const int lane = threadIdx.x & 31;
    const long row = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (row >= nrows) return;
    const int j = static_cast<int>((row / Hkv) % Skv);
    const long off = row * D;
    for (int d = 2 * lane; d < D; d += 64) {
        float x0 = load_as_f32(k + off + d), x1 = load_as_f32(k + off + d + 1);
        if (tab != nullptr) rot_pair(x0, x1, tab[static_cast<long>(j) * (D / 2) + d / 2], 1.f);
        Kf[off + d] = x0;
        Kf[off + d + 1] = x1;
        Vf[off + d] = load_as_f32(v + off + d);
        Vf[off + d + 1] = load_as_f32(v + off + d + 1);
    }
}

struct BwdParams {
    const float* Qf;     // [B, Sq, Hq, D]  rotated q
    const float* Kf;     // [B, Skv, Hkv, D] rotated k
    const float* Vf;     // [B, Skv, Hkv, D]
    const float* dOf;    // [B, Sq, Hq, D]
    const float* lse;    // [B, Hq, Sq]  natural-log logsumexp of the scaled scores
    const float* Dvec;   // [B, Hq, Sq]
    const float2* tab;   // (cos, sin) per [position][D/2], or null without RoPE
    float* g_f32;        // output gradient (fp32) or
    __nv_bfloat16* g_bf16;   // (bf16)
    int B, Hq, Hkv, Sq, Skv, q_pos0;
    int causal;
    float scale;
    const float* mask;       // additive mask of the forward or null; element strides below, rows of Skv
    long mask_bs, mask_hs;
};

// Sum over the 4 threads of a row (lanes 4r .. 4r+3 of the warp).
__device__ __forceinline__ float quad_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

template <int D>
__device__ __forceinline__ void store_grad(const BwdParams& p, long off, const float (&g)[D / 4]) {
    if (p.g_f32 != nullptr) {
#pragma unroll
        for (int e = 0; e < D / 4; e += 4)
            *reinterpret_cast<float4*>(p.g_f32 + off + e) = make_float4(g[e], g[e + 1], g[e + 2], g[e + 3]);
    } else {
#pragma unroll
        for (int e = 0; e < D / 4; e += 8)
            *reinterpret_cast<uint4*>(p.g_bf16 + off + e) =
                make_uint4(pack_bf16x2(g[e], g[e + 1]), pack_bf16x2(g[e + 2], g[e + 3]),
                           pack_bf16x2(g[e + 4], g[e + 5]), pack_bf16x2(g[e + 6], g[e + 7]));
    }
}

// dQ: CTA (row block, h, b); thread t: row r = t / 4 of the block, dims [(t%4) D/4, +D/4).
template <int D>
__global__ void __launch_bounds__(kBwdThreads) bwd_dq_kernel(const BwdParams p) {
    constexpr int DQ = D / 4;
    extern __shared__ float smem_f[];
    float* sK = smem_f;                     // [kBwdTile][D]
    float* sV = smem_f + kBwdTile * D;      // [kBwdTile][D]
    const int h = blockIdx.y, b = blockIdx.z;
    const int kvh = h / (p.Hq / p.Hkv);
    const int r = threadIdx.x >> 2, part = threadIdx.x & 3;
    const int i = blockIdx.x * kBwdRows + r;
    const bool live = i < p.Sq;
    const long qoff = ((static_cast<long>(b) * p.Sq + (live ? i : 0)) * p.Hq + h) * D + part * DQ;
    float qv[DQ], gv[DQ], acc[DQ];
#pragma unroll
    for (int e = 0; e < DQ; ++e) {
        qv[e] = live ? p.Qf[qoff + e] : 0.f;
        gv[e] = live ? p.dOf[qoff + e] : 0.f;
        acc[e] = 0.f;
    }
    const long srow = (static_cast<long>(b) * p.Hq + h) * p.Sq + (live ? i : 0);
    const float lse = live ? p.lse[srow] : -INFINITY;
    const float Dv = live ? p.Dvec[srow] : 0.f;
    const long off_c = static_cast<long>(p.Skv) - p.Sq;
    // keys this row may see: [0, nvis)
    long nvis = p.causal ? static_cast<long>(i) + off_c + 1 : p.Skv;
    nvis = nvis < 0 ? 0 : (nvis > p.Skv ? p.Skv : nvis);
    if (lse == -INFINITY) nvis = 0;   // a row without a visible key has no gradient
    // keys any row of this block may see
    const long last_row = static_cast<long>(blockIdx.x) * kBwdRows + kBwdRows - 1;
    long kmax = p.causal ? last_row + off_c + 1 : p.Skv;
    kmax = kmax < 0 ? 0 : (kmax > p.Skv ? p.Skv : kmax);
    for (long k0 = 0; k0 < kmax; k0 += kBwdTile) {
        __syncthreads();
        for (int w = threadIdx.x; w < kBwdTile * D / 4; w += kBwdThreads) {
            const int jj = w / (D / 4), c = (w % (D / 4)) * 4;
            const long j = k0 + jj;
            float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk;
            if (j < p.Skv) {
                const long koff = ((static_cast<long>(b) * p.Skv + j) * p.Hkv + kvh) * D + c;
                kk = *reinterpret_cast<const float4*>(p.Kf + koff);
                vv = *reinterpret_cast<const float4*>(p.Vf + koff);
            }
            *reinterpret_cast<float4*>(sK + jj * D + c) = kk;
            *reinterpret_cast<float4*>(sV + jj * D + c) = vv;
        }
        __syncthreads();
        const int jn = static_cast<int>(min(static_cast<long>(kBwdTile), kmax - k0));
        for (int jj = 0; jj < jn; ++jj) {
            const float* kr = sK + jj * D + part * DQ;
            const float* vr = sV + jj * D + part * DQ;
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int e = 0; e < DQ; ++e) {
                s = fmaf(qv[e], kr[e], s);
                dp = fmaf(gv[e], vr[e], dp);
            }
            s = quad_sum(s);
            dp = quad_sum(dp);
            const bool vis = k0 + jj < nvis;
            const float mval = (vis && p.mask != nullptr)
                                   ? p.mask[b * p.mask_bs + h * p.mask_hs + static_cast<long>(i) * p.Skv + k0 + jj]
                                   : 0.f;
            const float pr = vis ? __expf(s * p.scale + mval - lse) : 0.f;
            const float ds = pr * (dp - Dv) * p.scale;
#pragma unroll
            for (int e = 0; e < DQ; ++e) acc[e] = fmaf(ds, kr[e], acc[e]);
        }
    }
    if (!live) return;
    if (p.tab != nullptr) {
        const float2* t = p.tab + static_cast<long>(p.q_pos0 + i) * (D / 2) + part * (DQ / 2);
#pragma unroll
        for (int e = 0; e < DQ; e += 2) rot_pair(acc[e], acc[e + 1], t[e / 2], -1.f);
    }
    store_grad<D>(p, qoff, acc);
}

// dK, dV: CTA (key block, kvh, b); thread t: key j = block*64 + t/4, dims [(t%4) D/4, +D/4).
// Writes dK to p.g_* and dV to dv_f32 / dv_bf16.
template <int D>
__global__ void __launch_bounds__(kBwdThreads) bwd_dkdv_kernel(const BwdParams p, float* __restrict__ dv_f32,
                                                                __nv_bfloat16* __restrict__ dv_bf16) {
    constexpr int DQ = D / 4;
    extern __shared__ float smem_f[];
    float* sQ = smem_f;                        // [kBwdTile][D]
    float* sG = smem_f + kBwdTile * D;         // [kBwdTile][D]  dO
    float* sL = smem_f + 2 * kBwdTile * D;     // [kBwdTile] lse
    float* sD = sL + kBwdTile;                 // [kBwdTile] Dvec
    const int kvh = blockIdx.y, b = blockIdx.z;
    const int G = p.Hq / p.Hkv;
    const int r = threadIdx.x >> 2, part = threadIdx.x & 3;
    const int j = blockIdx.x * kBwdRows + r;
    const bool live = j < p.Skv;
    const long koff = ((static_cast<long>(b) * p.Skv + (live ? j : 0)) * p.Hkv + kvh) * D + part * DQ;
    float kv[DQ], vv[DQ], dk[DQ], dvv[DQ];
#pragma unroll
    for (int e = 0; e < DQ; ++e) {
        kv[e] = live ? p.Kf[koff + e] : 0.f;
        vv[e] = live ? p.Vf[koff + e] : 0.f;
        dk[e] = 0.f;
        dvv[e] = 0.f;
    }
    const long off_c = static_cast<long>(p.Skv) - p.Sq;
    // query rows that may see key j: i >= j - off_c; the block's first key bounds the tiles
    const long first_key = static_cast<long>(blockIdx.x) * kBwdRows;
    long i_lo = p.causal ? first_key - off_c : 0;
    i_lo = i_lo < 0 ? 0 : i_lo;
    const long i_start = (i_lo / kBwdTile) * kBwdTile;
    for (int hg = 0; hg < G; ++hg) {
        const int h = kvh * G + hg;
        for (long i0 = i_start; i0 < p.Sq; i0 += kBwdTile) {
            __syncthreads();
            for (int w = threadIdx.x; w < kBwdTile * D / 4; w += kBwdThreads) {
                const int ii = w / (D / 4), c = (w % (D / 4)) * 4;
                const long i = i0 + ii;
                float4 qq = make_float4(0.f, 0.f, 0.f, 0.f), gg = qq;
                if (i < p.Sq) {
                    const long qoff = ((static_cast<long>(b) * p.Sq + i) * p.Hq + h) * D + c;
                    qq = *reinterpret_cast<const float4*>(p.Qf + qoff);
                    gg = *reinterpret_cast<const float4*>(p.dOf + qoff);
                }
                *reinterpret_cast<float4*>(sQ + ii * D + c) = qq;
                *reinterpret_cast<float4*>(sG + ii * D + c) = gg;
            }
            for (int w = threadIdx.x; w < kBwdTile; w += kBwdThreads) {
                const long i = i0 + w;
                const long srow = (static_cast<long>(b) * p.Hq + h) * p.Sq + i;
                sL[w] = i < p.Sq ? p.lse[srow] : -INFINITY;
                sD[w] = i < p.Sq ? p.Dvec[srow] : 0.f;
            }
            __syncthreads();
            const int in = static_cast<int>(min(static_cast<long>(kBwdTile), static_cast<long>(p.Sq) - i0));
            for (int ii = 0; ii < in; ++ii) {
                const float* qr = sQ + ii * D + part * DQ;
                const float* gr = sG + ii * D + part * DQ;
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int e = 0; e < DQ; ++e) {
                    s = fmaf(kv[e], qr[e], s);
                    dp = fmaf(vv[e], gr[e], dp);
                }
                s = quad_sum(s);
                dp = quad_sum(dp);
                const long i = i0 + ii;
                const float lse = sL[ii];
                const bool vis = live && lse != -INFINITY && (!p.causal || static_cast<long>(j) <= i + off_c);
                const float mval = (vis && p.mask != nullptr)
                                       ? p.mask[b * p.mask_bs + h * p.mask_hs + i * p.Skv + j]
                                       : 0.f;
                const float pr = vis ? __expf(s * p.scale + mval - lse) : 0.f;
                const float ds = pr * (dp - sD[ii]) * p.scale;
#pragma unroll
                for (int e = 0; e < DQ; ++e) {
                    dvv[e] = fmaf(pr, gr[e], dvv[e]);
                    dk[e] = fmaf(ds, qr[e], dk[e]);
                }
            }
        }
    }
    if (!live) return;
    if (p.tab != nullptr) {
        const float2* t = p.tab + static_cast<long>(j) * (D / 2) + part * (DQ / 2);
#pragma unroll
        for (int e = 0; e < DQ; e += 2) rot_pair(dk[e], dk[e + 1], t[e / 2], -1.f);
    }
    store_grad<D>(p, koff, dk);
    BwdParams pv = p;
    pv.g_f32 = dv_f32;
    pv.g_bf16 = dv_bf16;
    store_grad<D>(pv, koff, dvv);
}

}  // namespace attn
