// decode.cuh -- split-KV flash-decode: one query token per (sequence, q head) against a cache.
//
// oxibonsai-model 0.1.4, src/layers/flash_decode.rs: the cache of a sequence is cut into
// contiguous near-equal key ranges ("tiles"; flash_decode_single_head gives the first L % n
// tiles one extra key), each range yields a normalised partial output and its logsumexp
// (flash_decode_tile), and the partials are merged with weights exp(lse_s - lse)
// (combine_tile_outputs, which drops ranges whose lse is -inf).  whisper-apr 0.3.1
// src/model/lfm2/gqa.rs, attention_cached: the new token attends to the whole cache, no mask,
// q head h reading kv head h / (Hq/Hkv).
//
// Split kernel: one CTA per (split, kv head x head block, sequence), 4 warps.  GC query heads of a
// group (GC = the whole group when it has at most 4 heads) are handled together so every K/V row
// is read from HBM once per GC heads; larger groups run G/GC CTAs that meet in L2.  A key row of one kv
// head is D bf16 = D*2 contiguous bytes; LPK = D/8 lanes read it with one 16-byte load each
// (coalesced: a warp load instruction covers 32/LPK whole rows).  Each lane keeps 8 dims of q for
// every head of the group and computes partial dot products for the rows it loaded; partials are
// reduce-scattered over the LPK lanes of a row with shuffles so that each lane ends with whole
// scores, exponentiated once, then gathered back for the P.V update.
//
// Combine kernel: one warp per (sequence, q head) merges the splits by logsumexp.
#pragma once

#include "common.cuh"

namespace attn {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeMinKeysPerSplit = 512;

// Number of splits sequence length L uses, and the key range of split s (near-equal contiguous
// chunks, the first L % n one key longer).
__host__ __device__ __forceinline__ int decode_num_splits(int L, int max_splits) {
    int n = L / kDecodeMinKeysPerSplit;
    if (n < 1) n = 1;
    if (n > max_splits) n = max_splits;
    return n;
}

__device__ __forceinline__ int clamp_seqlen(int L, int Smax) {
    if (L < 1 || L > Smax) {
        record_error(ATTN_DEVICE_ERR_SEQLEN);
        L = L < 1 ? 1 : Smax;
    }
    return L;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <int D, int G>   // G: query heads handled by one CTA
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_split_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
    const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ seqlens,
    float* __restrict__ o_part, float* __restrict__ lse_part, int Hkv, int group, int Smax,
    int max_splits, float scale_log2) {
    constexpr int LPK = D / 8;            // lanes per key row
    constexpr int SLOTS = 32 / LPK;       // rows per warp load instruction
    constexpr int NLOAD = 8;              // load instructions per tensor per iteration
    constexpr int KPW = NLOAD * SLOTS;    // keys per warp iteration
    constexpr int DUP = LPK / NLOAD;      // lanes ending with the same key's scores (1 or 2)
    static_assert(DUP >= 1, "head dim too small for this layout");

    extern __shared__ float sm_dec[];
    const int split = blockIdx.x, b = blockIdx.z;
    const int kvh = blockIdx.y / (group / G);
    const int h0 = kvh * group + (blockIdx.y % (group / G)) * G;   // first q head of this CTA
    const int L = clamp_seqlen(seqlens[b], Smax);
    const int nsplit = decode_num_splits(L, max_splits);
    if (split >= nsplit) return;
    const int base = L / nsplit, rem = L % nsplit;
    const int kbeg = split * base + (split < rem ? split : rem);
    const int kend = kbeg + base + (split < rem ? 1 : 0);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = lane % LPK, r = lane / LPK;
    const int Hq = Hkv * group;

    // q of the group, dims [8c, 8c+8), pre-scaled so that q.k is already in log2 units
    float qf[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint4 w = *reinterpret_cast<const uint4*>(q + (static_cast<long>(b) * Hq + h0 + g) * D + c * 8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            qf[g][2 * e] = bf16lo_to_f32(ww[e]) * scale_log2;
            qf[g][2 * e + 1] = bf16hi_to_f32(ww[e]) * scale_log2;
        }
    }

    float m[G], lsum[G], acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        lsum[g] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
    }

    const long row_stride = static_cast<long>(Hkv) * D;   // elements between consecutive keys
    const __nv_bfloat16* kbase = kc + (static_cast<long>(b) * Smax * Hkv + kvh) * D + c * 8;
    const __nv_bfloat16* vbase = vc + (static_cast<long>(b) * Smax * Hkv + kvh) * D + c * 8;

    for (int chunk = kbeg + warp * KPW; chunk < kend; chunk += kDecodeWarps * KPW) {
        uint4 kr[NLOAD], vr[NLOAD];
#pragma unroll
        for (int n = 0; n < NLOAD; ++n) {
            const int key = chunk + n * SLOTS + r;
            if (key < kend) {
                kr[n] = ldg_stream(kbase + key * row_stride);
                vr[n] = ldg_stream(vbase + key * row_stride);
            } else {
                kr[n] = make_uint4(0, 0, 0, 0);
                vr[n] = make_uint4(0, 0, 0, 0);
            }
        }
        // partial dot products over this lane's 8 dims
        float part[NLOAD][G];
#pragma unroll
        for (int n = 0; n < NLOAD; ++n) {
            const uint32_t ww[4] = {kr[n].x, kr[n].y, kr[n].z, kr[n].w};
            float kf[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                kf[2 * e] = bf16lo_to_f32(ww[e]);
                kf[2 * e + 1] = bf16hi_to_f32(ww[e]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) s = fmaf(qf[g][e], kf[e], s);
                part[n][g] = s;
            }
        }
        // reduce-scatter over the LPK lanes of a row: round k halves the set of keys a lane keeps
#pragma unroll
        for (int h = NLOAD / 2, off = LPK / 2; h >= 1; h /= 2, off /= 2) {
            const bool upper = (lane & off) != 0;
#pragma unroll
            for (int n = 0; n < h; ++n) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float send = upper ? part[n][g] : part[n + h][g];
                    const float keep = upper ? part[n + h][g] : part[n][g];
                    part[n][g] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            }
        }
#pragma unroll
        for (int off = DUP / 2; off >= 1; off /= 2)
#pragma unroll
            for (int g = 0; g < G; ++g) part[0][g] += __shfl_xor_sync(0xffffffffu, part[0][g], off);

        // this lane's whole scores: key n_own of the iteration, every head of the group
        const int n_own = c / DUP;
        const bool valid = chunk + n_own * SLOTS + r < kend;
        float t[G], mx[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            t[g] = valid ? part[0][g] : -INFINITY;
            mx[g] = t[g];
        }
#pragma unroll
        for (int off = LPK / 2; off >= 1; off /= 2)
#pragma unroll
            for (int g = 0; g < G; ++g) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], off));

        float p[G], corr[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float mn = fmaxf(m[g], mx[g]);
            corr[g] = (m[g] == -INFINITY) ? 0.f : fast_exp2(m[g] - mn);
            m[g] = mn;
            const float mu = (mn == -INFINITY) ? 0.f : mn;
            p[g] = fast_exp2(t[g] - mu);
            lsum[g] = lsum[g] * corr[g] + ((c % DUP) == 0 ? p[g] : 0.f);
        }
        // gather every key's weights and update the output dims this lane owns
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] *= corr[g];
#pragma unroll
        for (int n = 0; n < NLOAD; ++n) {
            const int src = r * LPK + n * DUP;
            const uint32_t ww[4] = {vr[n].x, vr[n].y, vr[n].z, vr[n].w};
            float vf[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                vf[2 * e] = bf16lo_to_f32(ww[e]);
                vf[2 * e + 1] = bf16hi_to_f32(ww[e]);
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float pn = __shfl_sync(0xffffffffu, p[g], src);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pn, vf[e], acc[g][e]);
            }
        }
    }

    // row sum of each slot
#pragma unroll
    for (int off = LPK / 2; off >= 1; off /= 2)
#pragma unroll
        for (int g = 0; g < G; ++g) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], off);

    // merge the (warp, slot) partial states of the CTA through shared memory
    constexpr int NPART = kDecodeWarps * SLOTS;
    float* sm_m = sm_dec;                       // [NPART][G]
    float* sm_l = sm_m + NPART * G;             // [NPART][G]
    float* sm_o = sm_l + NPART * G;             // [NPART][G][D]
    const int part_id = warp * SLOTS + r;
    if (c == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            sm_m[part_id * G + g] = m[g];
            sm_l[part_id * G + g] = lsum[g];
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) sm_o[(part_id * G + g) * D + c * 8 + e] = acc[g][e];
    __syncthreads();

    for (int w = threadIdx.x; w < G * D; w += blockDim.x) {
        const int g = w / D, d = w % D;
        float M = -INFINITY;
        for (int pi = 0; pi < NPART; ++pi) M = fmaxf(M, sm_m[pi * G + g]);
        float Ls = 0.f, Od = 0.f;
        if (M != -INFINITY) {
            for (int pi = 0; pi < NPART; ++pi) {
                const float mp = sm_m[pi * G + g];
                if (mp == -INFINITY) continue;
                const float wgt = fast_exp2(mp - M);
                Ls = fmaf(sm_l[pi * G + g], wgt, Ls);
                Od = fmaf(sm_o[(pi * G + g) * D + d], wgt, Od);
            }
        }
        const long hq = static_cast<long>(b) * Hq + h0 + g;
        const long slot = hq * max_splits + split;
        o_part[slot * D + d] = Ls > 0.f ? Od / Ls : 0.f;
        if (d == 0) lse_part[slot] = Ls > 0.f ? (M + fast_log2(Ls)) * 0.69314718055994531f : -INFINITY;
    }
}

// One warp per (sequence, q head): out = sum_s exp(lse_s - lse) o_s over splits with finite lse,
// lse = max + ln sum exp(lse_s - max).
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    const int32_t* __restrict__ seqlens, __nv_bfloat16* __restrict__ o, float* __restrict__ o_f32,
    float* __restrict__ lse, int B, int Hq, int Smax, int max_splits) {
    constexpr int DPL = D / 32;   // dims per lane
    const int warp_global = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (warp_global >= B * Hq) return;
    const int b = warp_global / Hq;
    int L = seqlens[b];
    if (L < 1) L = 1;
    if (L > Smax) L = Smax;
    const int nsplit = decode_num_splits(L, max_splits);
    const long slot0 = static_cast<long>(warp_global) * max_splits;

    float M = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, lse_part[slot0 + s]);
#pragma unroll
    for (int off = 16; off >= 1; off /= 2) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));

    float acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
    float total = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < nsplit; ++s) {
            const float ls = lse_part[slot0 + s];
            if (ls == -INFINITY) continue;
            const float w = __expf(ls - M);
            total += w;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, o_part[(slot0 + s) * D + lane * DPL + e], acc[e]);
        }
    }
    const float inv = total > 0.f ? 1.f / total : 0.f;
    if (o_f32 != nullptr) {
        float* orow = o_f32 + static_cast<long>(warp_global) * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; ++e) orow[e] = acc[e] * inv;
    } else {
        __nv_bfloat16* orow = o + static_cast<long>(warp_global) * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < DPL; e += 2)
            *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    }
    if (lse != nullptr && lane == 0) lse[warp_global] = total > 0.f ? M + logf(total) : -INFINITY;
}

}  // namespace attn
