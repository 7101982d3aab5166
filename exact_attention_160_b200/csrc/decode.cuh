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
// Split kernel: one CTA per (split, kv head x head block, sequence).  A producer warp streams the
// split's K and V rows (one kv head: D bf16 = 2D contiguous bytes per key) into a two-stage
// shared-memory ring with TMA; four consumer warps compute.  Up to 16 query heads of a group are
// handled together as the rows of 16x8x16 bf16 tensor-core MMAs (fp32 accumulation), so every
// K/V row is read from HBM once for the whole group and the dot products cost about one MMA per
// key instead of dozens of FMA, shuffle and conversion instructions -- which is what lets the
// kernel run at memory speed.  The S accumulators, exponentiated and rounded to bf16, are the A
// operand of O += P V directly (no shuffles).
//
// Combine kernel: one CTA per (sequence, q head) merges the splits by logsumexp.
#pragma once

#include "common.cuh"

namespace attn {

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

constexpr int kDecodeConsumerWarps = 4;
constexpr int kDecodeThreads = (kDecodeConsumerWarps + 1) * 32;   // + one TMA producer warp
constexpr int kDecodeStages = 2;
constexpr int kDecodeMaxHeads = 16;                                 // q heads per CTA (MMA rows)

// A tile is TK keys of one kv head: one 128-byte-swizzled TMA box per 64 dims, for K and for V
// (16 KB each).  Each consumer warp owns KW = TK/4 keys of the tile.
template <int D>
struct DecCfg {
    static constexpr int TK = (D == 64) ? 128 : 64;
    static constexpr int KW = TK / kDecodeConsumerWarps;     // keys per warp per tile
    static constexpr int NBOX = D / 64;
    static constexpr int BOX_BYTES = TK * 128;
    static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int RING_BYTES = kDecodeStages * STAGE_BYTES;
    static constexpr int SMEM_BYTES = RING_BYTES + 128 /* barriers */ + 1024 /* alignment */;
};

// Byte offset of the 16-byte chunk holding dims [8*ch, 8*ch+8) of row `row` in a tile made of
// 128-byte-swizzled boxes of 64 dims (TMA SWIZZLE_128B layout, 1024-byte aligned boxes).
template <int D>
__device__ __forceinline__ uint32_t dec_chunk(int row, int ch) {
    return static_cast<uint32_t>((ch >> 3) * DecCfg<D>::BOX_BYTES + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
}

// One CTA per (split, kv head x head block, sequence): warp 4 streams the split's K and V rows
// into a two-stage shared-memory ring with TMA; warps 0-3 each take a quarter of every tile.
// The group's query heads (up to 16) are the rows of 16x8x16 bf16 MMAs: S = Q K^T with the keys
// as MMA columns, then the S accumulators, exponentiated and rounded to bf16, are directly the
// A operand of O += P V.  Every K/V row is read from HBM once for all heads of the CTA.
template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_split_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ seqlens, float* __restrict__ o_part,
    float* __restrict__ lse_part, int Hkv, int group, int heads_per_cta, int Smax, int max_splits,
    float scale_log2) {
    using C = DecCfg<D>;
    constexpr int KW = C::KW;
    constexpr int NT = KW / 8;        // key columns of S per warp (8 keys each)
    constexpr int KS = D / 16;        // k steps of S = Q K^T
    constexpr int NKS = KW / 16;      // k steps of O += P V
    constexpr int ND = D / 8;         // dim columns of O
    extern __shared__ uint8_t sm_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_full = reinterpret_cast<uint64_t*>(ring + C::RING_BYTES);
    uint64_t* bar_empty = bar_full + kDecodeStages;

    const int split = blockIdx.x, b = blockIdx.z;
    const int GC = heads_per_cta;
    const int kvh = blockIdx.y / (group / GC);
    const int h0 = kvh * group + (blockIdx.y % (group / GC)) * GC;   // first q head of this CTA
    const int L = clamp_seqlen(seqlens[b], Smax);
    const int nsplit = decode_num_splits(L, max_splits);
    if (split >= nsplit) return;
    const int base = L / nsplit, rem = L % nsplit;
    const int kbeg = split * base + (split < rem ? split : rem);
    const int kend = kbeg + base + (split < rem ? 1 : 0);
    const int ntiles = (kend - kbeg + C::TK - 1) / C::TK;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecodeStages; ++s) {
            mbar_init(bar_full + s, 1);
            mbar_init(bar_empty + s, kDecodeConsumerWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();

    const int Hq = Hkv * group;
    const int g = lane >> 2, t4 = lane & 3;    // MMA fragment coordinates: row g, column pair t4
    float m_run = -INFINITY, l_run = 0.f, l_mma = 0.f;   // state of head row g (this lane's share)
    float o_acc[ND][4];                                   // O rows g (c0,c1) and g+8 (padding)
#pragma unroll
    for (int nd = 0; nd < ND; ++nd)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[nd][e] = 0.f;

    if (warp == kDecodeConsumerWarps) {
        // ------------------------------- TMA producer ----------------------------------
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();   // the cache is streamed once
            int issued = 0;
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % kDecodeStages;
                if (!mbar_wait(bar_empty + s, ((t / kDecodeStages) & 1) ^ 1)) break;
                mbar_arrive_expect_tx(bar_full + s, C::STAGE_BYTES);
                uint8_t* st = ring + s * C::STAGE_BYTES;
#pragma unroll
                for (int bx = 0; bx < C::NBOX; ++bx) {
                    tma_load_4d(&tm_k, bar_full + s, st + bx * C::BOX_BYTES, bx * 64, kvh, kbeg + t * C::TK, b, pol);
                    tma_load_4d(&tm_v, bar_full + s, st + C::TILE_BYTES + bx * C::BOX_BYTES, bx * 64, kvh,
                                kbeg + t * C::TK, b, pol);
                }
                issued = t + 1;
            }
            // no copy may still be landing when the ring is reused below
            for (int t = issued - kDecodeStages > 0 ? issued - kDecodeStages : 0; t < issued; ++t)
                mbar_wait(bar_full + t % kDecodeStages, (t / kDecodeStages) & 1);
        }
    } else {
        // ------------------------------- consumers -------------------------------------
        // A fragments of Q (rows = heads; rows >= GC and the padding rows 8-15 are zero)
        uint32_t qa[KS][2];
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            qa[kk][0] = 0;
            qa[kk][1] = 0;
            if (g < GC) {
                const uint32_t* qrow = reinterpret_cast<const uint32_t*>(q + (static_cast<long>(b) * Hq + h0 + g) * D);
                qa[kk][0] = qrow[(kk * 16 + 2 * t4) >> 1];
                qa[kk][1] = qrow[(kk * 16 + 8 + 2 * t4) >> 1];
            }
        }
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t % kDecodeStages;
            if (!__all_sync(0xffffffffu, mbar_wait(bar_full + s, (t / kDecodeStages) & 1))) { ok = false; break; }
            const uint32_t sK = smem_u32(ring + s * C::STAGE_BYTES);
            const uint32_t sV = sK + C::TILE_BYTES;
            const int r0 = warp * KW;                     // first tile row of this warp
            const int key0 = kbeg + t * C::TK + r0;       // its key index
            const int nvalid = kend - key0;               // keys [key0, key0 + nvalid) are real
            if (nvalid < KW) {
                // rows past the split end may hold anything (other data, NaN): zero their V so
                // that P = 0 times V stays 0 in the MMA
                uint8_t* vt = ring + s * C::STAGE_BYTES + C::TILE_BYTES;
                for (int idx = lane; idx < KW * (D / 8); idx += 32) {
                    const int rr = idx / (D / 8), ch = idx % (D / 8);
                    if (rr >= nvalid) *reinterpret_cast<uint4*>(vt + dec_chunk<D>(r0 + rr, ch)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();   // ordered before the stage's next TMA fill
                __syncwarp();
            }
            // S = Q K^T for this warp's KW keys: NT column blocks of 8 keys
            float sacc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
                for (int kk = 0; kk < KS; kk += 2) {
                    // matrices: (keys, dims 16kk+0..7), (.., +8..15), (.., 16kk+16..23), (.., +24..31)
                    const int row = r0 + nt * 8 + (lane & 7);
                    const int ch = 2 * kk + (lane >> 3);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(sK + dec_chunk<D>(row, ch), b0, b1, b2, b3);
                    mma_bf16_16816(sacc[nt], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
                    mma_bf16_16816(sacc[nt], qa[kk + 1][0], 0u, qa[kk + 1][1], 0u, b2, b3);
                }
            }
            // online softmax for head row g over the keys of this slice
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int kidx = nt * 8 + 2 * t4 + e;
                    const float v = kidx < nvalid ? sacc[nt][e] * scale_log2 : -INFINITY;
                    sacc[nt][e] = v;
                    mx = fmaxf(mx, v);
                }
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float mn = fmaxf(m_run, mx);
            const float corr = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - mn);
            m_run = mn;
            const float mu = (mn == -INFINITY) ? 0.f : mn;
            l_run *= corr;
            l_mma *= corr;
#pragma unroll
            for (int nd = 0; nd < ND; ++nd) {
                o_acc[nd][0] *= corr;
                o_acc[nd][1] *= corr;
            }
            uint32_t pa[NT];   // bf16 pairs of P for row g: keys (8nt + 2t4, +1)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const float p0 = fast_exp2(sacc[nt][0] - mu);
                const float p1 = fast_exp2(sacc[nt][1] - mu);
                l_run += p0 + p1;
                pa[nt] = pack_bf16x2(p0, p1);
                l_mma += bf16lo_to_f32(pa[nt]) + bf16hi_to_f32(pa[nt]);
            }
            // O += P V: k steps of 16 keys, dim columns of 8
#pragma unroll
            for (int ks = 0; ks < NKS; ++ks) {
#pragma unroll
                for (int nd = 0; nd < ND; nd += 2) {
                    // matrices (transposed): (keys 16ks+0..7, dims 8nd..), (keys +8..15, ..),
                    //                        (keys 16ks+0..7, dims 8nd+8..), (keys +8..15, ..)
                    const int row = r0 + ks * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                    const int ch = nd + (lane >> 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(sV + dec_chunk<D>(row, ch), b0, b1, b2, b3);
                    mma_bf16_16816(o_acc[nd], pa[2 * ks], 0u, pa[2 * ks + 1], 0u, b0, b1);
                    mma_bf16_16816(o_acc[nd + 1], pa[2 * ks], 0u, pa[2 * ks + 1], 0u, b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + s);
        }
        (void)ok;
        // row sums of head row g: add the four lanes t4 = 0..3
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
        l_mma += __shfl_xor_sync(0xffffffffu, l_mma, 1);
        l_mma += __shfl_xor_sync(0xffffffffu, l_mma, 2);
    }
    __syncthreads();   // every tile consumed, no copy in flight: the ring is reused for the merge

    // merge the four consumer warps' states per head row
    constexpr int NW = kDecodeConsumerWarps;
    float* sm_m = reinterpret_cast<float*>(ring);          // [NW][16]
    float* sm_l = sm_m + NW * kDecodeMaxHeads;             // [NW][16]
    float* sm_lm = sm_l + NW * kDecodeMaxHeads;            // [NW][16]
    float* sm_o = sm_lm + NW * kDecodeMaxHeads;            // [NW][16][D]
    static_assert((3 * NW * kDecodeMaxHeads + NW * kDecodeMaxHeads * D) * 4 <= C::RING_BYTES, "merge area");
    if (warp < NW) {
        if (t4 == 0) {
            sm_m[warp * kDecodeMaxHeads + g] = m_run;
            sm_l[warp * kDecodeMaxHeads + g] = l_run;
            sm_lm[warp * kDecodeMaxHeads + g] = l_mma;
        }
#pragma unroll
        for (int nd = 0; nd < ND; ++nd) {
            sm_o[(warp * kDecodeMaxHeads + g) * D + nd * 8 + 2 * t4] = o_acc[nd][0];
            sm_o[(warp * kDecodeMaxHeads + g) * D + nd * 8 + 2 * t4 + 1] = o_acc[nd][1];
        }
    }
    __syncthreads();
    for (int w = threadIdx.x; w < GC * D; w += blockDim.x) {
        const int hh = w / D, d = w % D;
        float M = -INFINITY;
        for (int pi = 0; pi < NW; ++pi) M = fmaxf(M, sm_m[pi * kDecodeMaxHeads + hh]);
        float Ls = 0.f, Lm = 0.f, Od = 0.f;
        if (M != -INFINITY) {
            for (int pi = 0; pi < NW; ++pi) {
                const float mp = sm_m[pi * kDecodeMaxHeads + hh];
                if (mp == -INFINITY) continue;
                const float wgt = fast_exp2(mp - M);
                Ls = fmaf(sm_l[pi * kDecodeMaxHeads + hh], wgt, Ls);
                Lm = fmaf(sm_lm[pi * kDecodeMaxHeads + hh], wgt, Lm);
                Od = fmaf(sm_o[(pi * kDecodeMaxHeads + hh) * D + d], wgt, Od);
            }
        }
        const long hq = static_cast<long>(b) * Hq + h0 + hh;
        const long slot = hq * max_splits + split;
        // normalised by the sum of the rounded weights the MMA used; lse from the fp32 sum
        o_part[slot * D + d] = Lm > 0.f ? Od / Lm : 0.f;
        if (d == 0) lse_part[slot] = Ls > 0.f ? (M + fast_log2(Ls)) * 0.69314718055994531f : -INFINITY;
    }
    // this CTA's partials are written: the combine grid may be scheduled (it still waits for
    // the whole grid to finish before it reads them)
    griddep_launch_dependents();
}

// One CTA of 256 threads per (sequence, q head): out = sum_s exp(lse_s - lse) o_s over splits
// with finite lse, lse = max + ln sum exp(lse_s - max) (the weights and their max go through
// shared memory; splits are handled kCombineChunk at a time).  Thread (d, g) accumulates output
// dim d over the splits s = g (mod 256/D), issuing independent coalesced loads, and the partial
// sums of the groups are added through shared memory.
constexpr int kCombineThreads = 256;
constexpr int kCombineChunk = 1024;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    const int32_t* __restrict__ seqlens, __nv_bfloat16* __restrict__ o, float* __restrict__ o_f32,
    float* __restrict__ lse, int B, int Hq, int Smax, int max_splits) {
    constexpr int NG = kCombineThreads / D;       // split groups
    __shared__ float sm_w[kCombineChunk];
    __shared__ float sm_red[kCombineThreads];
    __shared__ float sm_acc[NG][D];
    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int b = bh / Hq;
    int L = seqlens[b];
    if (L < 1) L = 1;
    if (L > Smax) L = Smax;
    const int nsplit = decode_num_splits(L, max_splits);
    const long slot0 = static_cast<long>(bh) * max_splits;
    // launched as a programmatic dependent of the split kernel: its partials are complete and
    // visible only after this wait
    griddep_wait();

    // global max of the split lse values
    float M = -INFINITY;
    for (int s = tid; s < nsplit; s += kCombineThreads) M = fmaxf(M, lse_part[slot0 + s]);
    sm_red[tid] = M;
    __syncthreads();
    for (int w = kCombineThreads / 2; w >= 1; w /= 2) {
        if (tid < w) sm_red[tid] = fmaxf(sm_red[tid], sm_red[tid + w]);
        __syncthreads();
    }
    M = sm_red[0];
    __syncthreads();

    const int d = tid % D, g = tid / D;
    float acc = 0.f, wsum = 0.f;
    for (int c0 = 0; c0 < nsplit; c0 += kCombineChunk) {
        const int cn = min(kCombineChunk, nsplit - c0);
        for (int s = tid; s < cn; s += kCombineThreads) {
            const float ls = lse_part[slot0 + c0 + s];
            sm_w[s] = (M == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - M);
        }
        __syncthreads();
#pragma unroll 8
        for (int s = g; s < cn; s += NG) {
            const float w = sm_w[s];
            acc = fmaf(w, o_part[(slot0 + c0 + s) * D + d], acc);
            wsum += w;
        }
        __syncthreads();
    }
    sm_acc[g][d] = acc;
    sm_red[tid] = wsum;
    __syncthreads();
    if (tid >= D) return;
    float a = 0.f, total = 0.f;
#pragma unroll
    for (int k = 0; k < NG; ++k) {
        a += sm_acc[k][d];
        total += sm_red[k * D + d];   // group k's weight sum (equal for every d of the group)
    }
    const float out = total > 0.f ? a / total : 0.f;
    if (o_f32 != nullptr) {
        o_f32[static_cast<long>(bh) * D + d] = out;
    } else {
        o[static_cast<long>(bh) * D + d] = __float2bfloat16_rn(out);
    }
    if (lse != nullptr && d == 0) lse[bh] = total > 0.f ? M + logf(total) : -INFINITY;
}

// The combine for at most kDecodeWarpCombineSplits splits: one warp per (sequence, q head), split
// s in lane s for the logsumexp weights and D / 32 output dims per lane, every load of the row
// issued before any result is used (one memory round trip, no shared memory or block barriers).
constexpr int kDecodeWarpCombineSplits = 16;
constexpr int kDecodeWarpCombineThreads = 256;

template <int D>
__global__ void __launch_bounds__(kDecodeWarpCombineThreads) decode_combine_warp_kernel(
    const float* __restrict__ o_part, const float* __restrict__ lse_part,
    const int32_t* __restrict__ seqlens, __nv_bfloat16* __restrict__ o, float* __restrict__ o_f32,
    float* __restrict__ lse, int B, int Hq, int Smax, int max_splits) {
    constexpr int E = D / 32;   // output dims per lane
    const long bh = static_cast<long>(blockIdx.x) * (kDecodeWarpCombineThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    griddep_wait();   // the split grid's partials are complete and visible after this
    if (bh >= static_cast<long>(B) * Hq) return;   // whole warps leave together
    const int b = static_cast<int>(bh / Hq);
    int L = seqlens[b];   // clamped as the split kernel does (which reports the clamp)
    L = L < 1 ? 1 : (L > Smax ? Smax : L);
    const int nsplit = decode_num_splits(L, max_splits);
    const long slot0 = bh * max_splits;
    const float ls = lane < nsplit ? lse_part[slot0 + lane] : -INFINITY;
    float x[kDecodeWarpCombineSplits][E];
#pragma unroll
    for (int sp = 0; sp < kDecodeWarpCombineSplits; ++sp) {
        if (sp < nsplit) {
            const float* src = o_part + (slot0 + sp) * D + lane * E;
            if constexpr (E == 2) {
                const float2 v = *reinterpret_cast<const float2*>(src);
                x[sp][0] = v.x, x[sp][1] = v.y;
            } else {
                const float4 v = *reinterpret_cast<const float4*>(src);
                x[sp][0] = v.x, x[sp][1] = v.y, x[sp][2] = v.z, x[sp][3] = v.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) x[sp][e] = 0.f;
        }
    }
    float M = ls;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, w));
    const float wt = (M == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - M);
    float total = wt;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) total += __shfl_xor_sync(0xffffffffu, total, w);
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
    for (int sp = 0; sp < kDecodeWarpCombineSplits; ++sp) {
        const float ws = __shfl_sync(0xffffffffu, wt, sp);   // 0 for sp >= nsplit
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(ws, x[sp][e], acc[e]);
    }
    const float inv = total > 0.f ? 1.f / total : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float out = acc[e] * inv;
        if (o_f32 != nullptr)
            o_f32[bh * D + lane * E + e] = out;
        else
            o[bh * D + lane * E + e] = __float2bfloat16_rn(out);
    }
    if (lse != nullptr && lane == 0) lse[bh] = total > 0.f ? M + logf(total) : -INFINITY;
}

}  // namespace attn
