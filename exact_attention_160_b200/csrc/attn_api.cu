// attn_api.cu -- the C ABI declared in include/attn_b200.h: host-side validation, TMA descriptor
// encoding and kernel launches.  No function here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <set>
#include <utility>

#include "../../include/attn_b200.h"
#include "common.cuh"
#include "decode.cuh"
#include "prefill_f32.cuh"
#include "prefill_tc.cuh"
#include "rope.cuh"
#include "backward.cuh"
#include "backward_mma.cuh"
#include "backward_tc.cuh"

using namespace attn;

namespace {

// Description of the most recent ATTN_ERR_CUDA of the calling thread.
thread_local char g_last_error[256] = "";

attn_status cuda_failure(const char* what, const char* detail) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, detail);
    return ATTN_ERR_CUDA;
}

// ------------------------------------------------------------------------------------------
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda)
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tensor [B][S][H][D] bf16 viewed as 4-D (D, H, S, B); box = 64 elements x 1 head x `rows` rows,
// 128-byte swizzle (the UMMA SW128 K-major / MN-major operand layout, and a bank-conflict-free
// ldmatrix layout).  Rows past S read as 0.
bool make_tmap_bshd_rows(CUtensorMap* m, const void* ptr, int B, int S, int H, int D, int rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        cuda_failure("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", "entry point unavailable");
        return false;
    }
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
    cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[96];
        snprintf(buf, sizeof(buf), "CUresult %d (dims %d,%d,%d,%d)", static_cast<int>(r), D, H, S, B);
        cuda_failure("cuTensorMapEncodeTiled", buf);
    }
    return r == CUDA_SUCCESS;
}

bool make_tmap_bshd(CUtensorMap* m, const void* ptr, int B, int S, int H, int D) {
    return make_tmap_bshd_rows(m, ptr, B, S, H, D, 128);
}

// Additive fp32 mask viewed as [Bm][Hm][Sq][Skv] (Bm = 1 or Hm = 1 where the strides broadcast)
// for TMA loads of 32-key x 128-row boxes with the 128-byte swizzle.  Returns false, with no
// error recorded, when the encoder refuses the view (the caller then reads the mask per row).
bool make_tmap_mask(CUtensorMap* m, const float* ptr, int B, int Hq, int Sq, int Skv, long bs, long hs) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t row = static_cast<cuuint64_t>(Skv) * 4;
    const cuuint64_t plane = row * static_cast<cuuint64_t>(Sq);
    const cuuint64_t hstride = hs ? static_cast<cuuint64_t>(hs) * 4 : plane;
    const cuuint64_t Hm = hs ? Hq : 1, Bm = bs ? B : 1;
    const cuuint64_t bstride = bs ? static_cast<cuuint64_t>(bs) * 4 : hstride * Hm;
    cuuint64_t dims[4] = {(cuuint64_t)Skv, (cuuint64_t)Sq, Hm, Bm};
    cuuint64_t strides[3] = {row, hstride, bstride};
    cuuint32_t box[4] = {32, 128, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output [B][S][H][D] (fp32 or bf16) for TMA stores of 32-column x 128-row boxes: 128-byte rows
// with the 128-byte swizzle (fp32) or 64-byte rows with the 64-byte swizzle (bf16).
bool make_tmap_out(CUtensorMap* m, void* ptr, int B, int S, int H, int D, bool f32) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        cuda_failure("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", "entry point unavailable");
        return false;
    }
    const cuuint64_t es = f32 ? 4 : 2;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es, (cuuint64_t)S * H * D * es};
    cuuint32_t box[4] = {32, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, ptr, dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[96];
        snprintf(buf, sizeof(buf), "CUresult %d (out dims %d,%d,%d,%d)", static_cast<int>(r), D, H, S, B);
        cuda_failure("cuTensorMapEncodeTiled", buf);
    }
    return r == CUDA_SUCCESS;
}

// fp32 array [rows][cols] viewed 2-D with a box of 128 columns x 1 row, no swizzle; columns past
// `cols` read as 0.  The row stride (cols * 4 bytes) must be a multiple of 16.
bool make_tmap_rows_f32(CUtensorMap* m, const void* ptr, long rows, int cols) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) {
        cuda_failure("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", "entry point unavailable");
        return false;
    }
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
    cuuint32_t box[2] = {128, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[96];
        snprintf(buf, sizeof(buf), "CUresult %d (rows %ld, cols %d)", static_cast<int>(r), rows, cols);
        cuda_failure("cuTensorMapEncodeTiled", buf);
    }
    return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Status of the launch just made (clears the runtime's launch error so it is not reported twice).
attn_status launch_status(const char* what) {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ATTN_OK : cuda_failure(what, cudaGetErrorString(e));
}

// Kernel attributes belong to the kernel's image on one device, so each (device, kernel) pair
// is configured once, on its first launch from that device.  With min_regs > 0 the kernel is
// first checked to be compiled with at least that many registers per thread.
std::mutex g_attr_mu;
std::set<std::pair<int, const void*>> g_attr_done;

attn_status prepare_kernel(const void* fn, int smem_bytes, const char* name, int min_regs = 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_failure("cudaGetDevice", cudaGetErrorString(e));
    const std::pair<int, const void*> key(dev, fn);
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (g_attr_done.count(key) != 0) return ATTN_OK;
    if (min_regs > 0) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, fn);
        if (e != cudaSuccess) return cuda_failure(name, cudaGetErrorString(e));
        if (fa.numRegs < min_regs) {
            char buf[96];
            snprintf(buf, sizeof(buf), "compiled with %d registers per thread, needs %d", fa.numRegs, min_regs);
            cuda_failure(name, buf);
            return ATTN_ERR_UNSUPPORTED;
        }
    }
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return cuda_failure(name, cudaGetErrorString(e));
    g_attr_done.insert(key);
    return ATTN_OK;
}

attn_status check_common(int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || D <= 0) return ATTN_ERR_INVALID_ARG;
    if (Skv == 0) return ATTN_ERR_EMPTY_KV;
    if (Skv < 0) return ATTN_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ATTN_ERR_DIM_MISMATCH;
    if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// Head dims other than 64 and 128 run at Dp = 64 (D < 64) or 128 (64 < D < 128) with q, k, v
// (and dout) zero-padded in the workspace: padded dims add nothing to q.k, the caller's scale is
// kept, RoPE keeps the frequencies of D (padding pairs rotate by the identity), and the outputs
// are copied back without the padding.  D must be even (whole 32-bit words per bf16 row).
bool native_dim(int D) { return D == 64 || D == 128; }
int padded_dim(int D) { return D <= 64 ? 64 : 128; }
bool paddable_dim(int D) { return D > 0 && D < 128 && !native_dim(D) && D % 2 == 0; }

attn_status launch_pad(const void* src, void* dst, long rows, int src_bytes, int dst_bytes, bool unpad,
                       cudaStream_t st) {
    const int sw = src_bytes / 4, dw = dst_bytes / 4;
    const long n = rows * dw;
    const unsigned grid = static_cast<unsigned>((n + 255) / 256 < 148L * 32 ? (n + 255) / 256 : 148L * 32);
    if (unpad)
        unpad_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), rows,
                                                sw, dw);
    else
        pad_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), rows, sw,
                                              dw);
    return launch_status(unpad ? "unpad_rows_kernel" : "pad_rows_kernel");
}

// Additive mask on the scaled scores: element (b, h, i, j) at ptr[b*bs + h*hs + i*Skv + j].
struct MaskArg {
    const float* ptr = nullptr;
    long bs = 0, hs = 0;
};

// Layout of the attn_fwd_ex workspace: rope table, then (bf16) rotated K as hi and lo halves.
constexpr int kNumSms = 148;   // B200

// Key splits of the tensor-core forward.  A bf16 problem whose query tiles fill at most half of
// the SMs divides each tile's key tiles among up to kMaxKvSplits CTAs (at least two key tiles
// each), so that the whole GPU works on it; the partials are merged by prefill_combine_kernel.
// A split is taken only when it shortens each CTA's key loop by at least kMinSplitSaving key
// tiles: the merge costs about as much as that (measured on B200: the Whisper-encoder shape, 12
// key tiles, runs 1.7 us faster unsplit than in 2 splits + merge).  Depends on the sizes only, so
// the workspace query and the launch agree.
constexpr int kMinSplitSaving = 8;
int fwd_kv_splits(int B, int Hq, int Sq, int Skv, attn_dtype dtype) {
    if (dtype == ATTN_FP32) return 1;
    const long tiles = static_cast<long>((Sq + 127) / 128) * B * Hq;
    if (tiles > kNumSms / 2) return 1;
    long n = kNumSms / tiles;
    const long nkv = (static_cast<long>(Skv) + 127) / 128;
    if (n > nkv / 2) n = nkv / 2;
    if (n > kMaxKvSplits) n = kMaxKvSplits;
    if (n < 2) return 1;
    const long saved = nkv - (nkv + n - 1) / n;   // key tiles the longest chunk is spared
    return saved >= kMinSplitSaving ? static_cast<int>(n) : 1;
}

// RoPE form of the bf16 forward: K rotated once beforehand into hi + lo halves that every CTA
// then reads (the default), or rotated inside the prefill kernel by two warps of each CTA as its
// tiles land (ATTN_ROPE_K_FORM=fused in the environment, read at every call).  Every K tile is
// read by about ceil(Sq / 128) * G / 2 CTAs; the in-kernel form repeats its rotation that many
// times and, measured on B200, is slower on every shape tried (GQA 32/8 causal, B2 S4096 D64:
// 648 vs 359 us; Sq 128 against Skv 8192: 105 vs 75 us), because two warps rotating 128 keys per
// tile fall behind the tile pipeline.  It is kept for that comparison.
bool rope_k_fused() {
    const char* f = getenv("ATTN_ROPE_K_FORM");
    return f != nullptr && strcmp(f, "fused") == 0;
}

// Workspace of attn_fwd_ex: with RoPE the cos/sin table and the rotated K as hi/lo bf16 halves;
// with key splits the fp32 partial O and logsumexp of every split.
struct ExWorkspace {
    size_t tab_off, khi_off, klo_off, opart_off, lpart_off, total;
    int positions;
    int splits;
};

ExWorkspace ex_workspace(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype, bool rope, int q_pos0) {
    ExWorkspace w{};
    size_t end = 0;
    if (rope) {
        long pq = static_cast<long>(q_pos0) + Sq;
        w.positions = static_cast<int>(pq > Skv ? pq : Skv);
        w.tab_off = 0;
        size_t tab = static_cast<size_t>(w.positions) * (D / 2) * sizeof(float2);
        w.khi_off = round_up(tab, 256);
        size_t kbytes = dtype != ATTN_FP32 ? static_cast<size_t>(B) * Skv * Hkv * D * 2 : 0;
        w.klo_off = round_up(w.khi_off + kbytes, 256);
        end = round_up(w.klo_off + kbytes, 256);
    }
    w.splits = fwd_kv_splits(B, Hq, Sq, Skv, dtype);
    if (w.splits > 1) {
        const size_t rows = static_cast<size_t>(B) * Sq * Hq;
        w.opart_off = end;
        w.lpart_off = round_up(w.opart_off + w.splits * rows * D * sizeof(float), 256);
        end = round_up(w.lpart_off + w.splits * rows * sizeof(float), 256);
    }
    w.total = end;
    return w;
}

template <int D, int ROPE>
attn_status launch_tc(const void* q, const void* k, const void* klo, const void* v, void* o, bool o_f32, float* lse,
                      int B, int Hq, int Hkv, int Sq, int Skv, float scale, int causal, const float2* tab, int q_pos0,
                      cudaStream_t st, MaskArg mk, int splits, float* o_part, float* lse_part) {
    CUtensorMap tq, tk, tkl, tv;
    if (!make_tmap_bshd(&tq, q, B, Sq, Hq, D) || !make_tmap_bshd(&tk, k, B, Skv, Hkv, D) ||
        !make_tmap_bshd(&tv, v, B, Skv, Hkv, D) || !make_tmap_bshd(&tkl, ROPE == kRopeKSplit ? klo : k, B, Skv, Hkv, D))
        return ATTN_ERR_CUDA;   // g_last_error set by make_tmap_bshd
    TcParams p{};
    p.o = o_f32 ? nullptr : static_cast<__nv_bfloat16*>(o);
    p.o_f32 = o_f32 ? static_cast<float*>(o) : nullptr;
    p.lse = lse;
    p.rope_tab = tab;
    p.B = B, p.Hq = Hq, p.Hkv = Hkv, p.Sq = Sq, p.Skv = Skv;
    p.causal = causal;
    const int G = Hq / Hkv;
    p.pair_heads = (G % 2 == 0) ? 1 : 0;
    p.n_row_tiles = p.pair_heads ? (Sq + 127) / 128 : (Sq + 255) / 256;
    p.heads_per_item = p.pair_heads ? Hq / 2 : Hq;
    // A problem so small that even one query tile per CTA fits in one wave of the 148 SMs runs
    // that way: twice the CTAs of the paired decomposition, each SM's exponentials spent on one
    // tile.  (When the single tiles would need a second wave, the pairs' shared K/V loads win.)
    if (static_cast<long>((Sq + 127) / 128) * B * Hq <= 148) {
        p.single_tile = 1;
        p.pair_heads = 0;
        p.n_row_tiles = (Sq + 127) / 128;
        p.heads_per_item = Hq;
    }
    p.q_pos0 = q_pos0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.mask = mk.ptr;
    p.mask_bs = mk.bs;
    p.mask_hs = mk.hs;
    p.inv_scale = 1.f / scale;
    p.mask_vec4 = mk.ptr != nullptr && aligned16(mk.ptr) && Skv % 4 == 0 && mk.bs % 4 == 0 && mk.hs % 4 == 0;
    p.kv_splits = 1;
    if (splits > 1) {
        if (!p.single_tile || splits > kMaxKvSplits || !o_part || !lse_part) return ATTN_ERR_UNSUPPORTED;
        p.kv_splits = splits;
        p.o_part = o_part;
        p.lse_part = lse_part;
    }
    const long grid = static_cast<long>(p.n_row_tiles) * B * p.heads_per_item * p.kv_splits;
    if (grid > 2147483647L) return ATTN_ERR_UNSUPPORTED;
    // The masked kernel is a separate instantiation, so the unmasked one carries no mask code.
    // Single query tiles at D = 64 run with interleaved keys: the CTA's two softmax warpgroups
    // take alternate key tiles of its one query tile, so that one works while the tensor core
    // serves the other (at D = 128 the ring has too few stages for the pair).
    auto kern = mk.ptr != nullptr ? prefill_tc_kernel<D, ROPE, true, false> : prefill_tc_kernel<D, ROPE, false, false>;
    // Their output (or a key split's fp32 partial) leaves through TMA stores; the other kernels
    // store from the threads and take the query map in that argument's place.
    CUtensorMap to = tq;
    if constexpr (D == 64) {
        if (p.single_tile) {
            kern = mk.ptr != nullptr ? prefill_tc_kernel<D, ROPE, true, true> : prefill_tc_kernel<D, ROPE, false, true>;
            const bool ok = p.kv_splits > 1 ? make_tmap_out(&to, o_part, p.kv_splits * B, Sq, Hq, D, true)
                                            : make_tmap_out(&to, o, B, Sq, Hq, D, o_f32);
            if (!ok) return ATTN_ERR_CUDA;
        }
    }
    // Masked D=64 without RoPE: the mask arrives by TMA when its rows are 16-byte aligned (the
    // kernel's smem holds the boxes either way; otherwise its threads read the mask per row).
    CUtensorMap tmk = tq;
    if constexpr (TcCfg<D, ROPE, true>::MASK_TMA)
        p.mask_tma = mk.ptr != nullptr && p.mask_vec4 &&
                     make_tmap_mask(&tmk, mk.ptr, B, Hq, Sq, Skv, mk.bs, mk.hs) ? 1 : 0;
    const int smem_bytes = mk.ptr != nullptr ? TcCfg<D, ROPE, true>::SMEM_BYTES : TcCfg<D, ROPE, false>::SMEM_BYTES;
    // The warpgroups re-split the launch's registers with setmaxnreg; a launch that holds fewer
    // than the split asks for would stall in setmaxnreg.inc, so such a build is refused.
    attn_status ps = prepare_kernel(reinterpret_cast<const void*>(kern), smem_bytes, "prefill_tc_kernel set-up",
                                    kTcLaunchRegsMin);
    if (ps != ATTN_OK) return ps;
    kern<<<static_cast<unsigned>(grid), kTcThreads, smem_bytes, st>>>(tq, tk, tkl, tv, to, tmk, p);
    attn_status s = launch_status("prefill_tc_kernel");
    if (s != ATTN_OK || p.kv_splits == 1) return s;
    // merge of the key splits, a programmatic dependent launch (it waits for the split grid)
    const long rows = static_cast<long>(B) * Sq * Hq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((rows + kPcThreads / 32 - 1) / (kPcThreads / 32)));
    cfg.blockDim = dim3(kPcThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, prefill_combine_kernel<D>, static_cast<const float*>(o_part),
                                             static_cast<const float*>(lse_part),
                                             o_f32 ? nullptr : static_cast<__nv_bfloat16*>(o),
                                             o_f32 ? static_cast<float*>(o) : nullptr, lse, B, Sq, Hq, splits);
    if (e != cudaSuccess) return cuda_failure("prefill_combine_kernel launch", cudaGetErrorString(e));
    return launch_status("prefill_combine_kernel");
}

template <int D>
attn_status launch_f32(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int Sq, int Skv, float scale, int causal, const float2* tab, int q_pos0, cudaStream_t st,
                       MaskArg mk) {
    const size_t smem = 2 * 64 * D * sizeof(float);
    auto kern = prefill_f32_kernel<D>;
    const attn_status ps = prepare_kernel(reinterpret_cast<const void*>(kern), static_cast<int>(smem),
                                          "cudaFuncSetAttribute(prefill_f32_kernel)");
    if (ps != ATTN_OK) return ps;
    dim3 grid((Sq + 63) / 64, Hq, B);
    if (grid.y > 65535 || grid.z > 65535) return ATTN_ERR_UNSUPPORTED;
    kern<<<grid, 256, smem, st>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                  static_cast<const float*>(v), static_cast<float*>(o), lse, Hq, Hkv, Sq, Skv, scale,
                                  causal, tab, q_pos0, mk.ptr, mk.bs, mk.hs);
    return launch_status("prefill_f32_kernel");
}

attn_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                     int Sq, int Skv, int D, float scale, int causal, attn_dtype dtype, float rope_base, int q_pos0,
                     void* workspace, size_t workspace_bytes, cudaStream_t st, int rope_dim, MaskArg mk = MaskArg{}) {
    attn_status s = check_common(B, Hq, Hkv, Sq, Skv, D, scale, causal);
    if (s != ATTN_OK) return s;
    if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP32 && dtype != ATTN_BF16_OUT_F32) return ATTN_ERR_INVALID_ARG;
    const bool o_f32 = dtype == ATTN_BF16_OUT_F32;
    const bool rope = rope_base > 0.f;
    if (rope && !isfinite(rope_base)) return ATTN_ERR_INVALID_ARG;
    if (rope && q_pos0 < 0) return ATTN_ERR_INVALID_ARG;
    if (rope && (D % 2) != 0) return ATTN_ERR_DIM_MISMATCH;

    const float2* tab = nullptr;
    // The workspace is required with RoPE; without it, a caller's workspace (attn_fwd_ex) turns on
    // the key splits of a small problem, and attn_fwd (none) runs it unsplit.
    const ExWorkspace w = ex_workspace(B, Hq, Hkv, Sq, Skv, D, dtype, rope, q_pos0);
    const int splits = (rope || workspace != nullptr) ? w.splits : 1;
    if ((rope || splits > 1) && (!workspace || workspace_bytes < w.total || !aligned16(workspace)))
        return ATTN_ERR_WORKSPACE;
    float* o_part = splits > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.opart_off) : nullptr;
    float* lse_part = splits > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.lpart_off) : nullptr;
    if (rope) {
        uint8_t* ws = static_cast<uint8_t*>(workspace);
        float2* t = reinterpret_cast<float2*>(ws + w.tab_off);
        const long n = static_cast<long>(w.positions) * (D / 2);
        rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0, st>>>(
            t, w.positions, D, static_cast<double>(rope_base), rope_dim);
        if ((s = launch_status("rope_table_kernel")) != ATTN_OK) return s;
        tab = t;
    }

    if (dtype == ATTN_FP32) {
        return D == 64 ? launch_f32<64>(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, scale, causal, tab, q_pos0, st, mk)
                       : launch_f32<128>(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, scale, causal, tab, q_pos0, st, mk);
    }
    if (!rope) {
        return D == 64 ? launch_tc<64, kRopeNone>(q, k, nullptr, v, o, o_f32, lse, B, Hq, Hkv, Sq, Skv, scale, causal,
                                              nullptr, 0, st, mk, splits, o_part, lse_part)
                       : launch_tc<128, kRopeNone>(q, k, nullptr, v, o, o_f32, lse, B, Hq, Hkv, Sq, Skv, scale, causal,
                                               nullptr, 0, st, mk, splits, o_part, lse_part);
    }
    if (rope_k_fused()) {
        // K rotated inside the prefill kernel as its tiles land
        return D == 64 ? launch_tc<64, kRopeKFused>(q, k, nullptr, v, o, o_f32, lse, B, Hq, Hkv, Sq, Skv, scale, causal,
                                                    tab, q_pos0, st, mk, splits, o_part, lse_part)
                       : launch_tc<128, kRopeKFused>(q, k, nullptr, v, o, o_f32, lse, B, Hq, Hkv, Sq, Skv, scale,
                                                     causal, tab, q_pos0, st, mk, splits, o_part, lse_part);
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* khi = reinterpret_cast<uint32_t*>(ws + w.khi_off);
    uint32_t* klo = reinterpret_cast<uint32_t*>(ws + w.klo_off);
    const long npairs = static_cast<long>(B) * Skv * Hkv * (D / 2);
    const long nchunks = npairs / 4;
    if (D % 8 == 0 && aligned16(k) && nchunks < (1L << 30)) {
        rope_split_kv_vec_kernel<<<static_cast<unsigned>((nchunks + 255) / 256 < 148 * 32 ? (nchunks + 255) / 256 : 148 * 32),
                                   256, 0, st>>>(static_cast<const uint4*>(k), reinterpret_cast<uint4*>(khi),
                                                 reinterpret_cast<uint4*>(klo), reinterpret_cast<const float4*>(tab),
                                                 static_cast<int>(nchunks), Skv, Hkv, D);
    } else {
        rope_split_kv_kernel<<<static_cast<unsigned>((npairs + 255) / 256 < 148 * 64 ? (npairs + 255) / 256 : 148 * 64),
                               256, 0, st>>>(static_cast<const uint32_t*>(k), khi, klo, tab, npairs, Skv, Hkv, D);
    }
    if ((s = launch_status("rope_split_kv_kernel")) != ATTN_OK) return s;
    return D == 64 ? launch_tc<64, kRopeKSplit>(q, khi, klo, v, o, o_f32, lse, B, Hq, Hkv, Sq, Skv, scale, causal, tab,
                                         q_pos0, st, mk, splits, o_part, lse_part)
                   : launch_tc<128, kRopeKSplit>(q, khi, klo, v, o, o_f32, lse, B, Hq, Hkv, Sq, Skv, scale, causal, tab,
                                          q_pos0, st, mk, splits, o_part, lse_part);
}

template <int D>
attn_status launch_decode(const void* q, const void* kc, const void* vc, const int32_t* seqlens, void* o, bool o_f32,
                          float* lse, int B, int Hq, int Hkv, int Smax, float scale, int num_splits, float* o_part,
                          float* lse_part, cudaStream_t st) {
    using C = DecCfg<D>;
    CUtensorMap tk, tv;
    if (!make_tmap_bshd_rows(&tk, kc, B, Smax, Hkv, D, C::TK) || !make_tmap_bshd_rows(&tv, vc, B, Smax, Hkv, D, C::TK))
        return ATTN_ERR_CUDA;
    const int G = Hq / Hkv;
    // heads per CTA: the largest power of two <= 16 dividing the group size
    int GC = 16;
    while (G % GC != 0) GC >>= 1;
    dim3 grid(num_splits, Hkv * (G / GC), B);
    if (grid.y > 65535 || grid.z > 65535) return ATTN_ERR_UNSUPPORTED;
    auto kern = decode_split_kernel<D>;
    const attn_status ps = prepare_kernel(reinterpret_cast<const void*>(kern), C::SMEM_BYTES,
                                          "cudaFuncSetAttribute(decode_split_kernel)");
    if (ps != ATTN_OK) return ps;
    kern<<<grid, kDecodeThreads, C::SMEM_BYTES, st>>>(tk, tv, static_cast<const __nv_bfloat16*>(q), seqlens, o_part,
                                                      lse_part, Hkv, G, GC, Smax, num_splits,
                                                      scale * 1.4426950408889634f);
    attn_status s = launch_status("decode_split_kernel");
    if (s != ATTN_OK) return s;
    // The combine is a programmatic dependent launch: its CTAs may be scheduled while the last
    // split CTAs finish, which hides the launch gap; it waits (griddepcontrol.wait) for the
    // split grid to complete before reading the partials.
    // Up to kDecodeWarpCombineSplits splits, one warp merges a (sequence, head) with all its
    // loads in flight; more splits take the block-per-head kernel, which walks them in chunks.
    const bool warp_combine = num_splits <= kDecodeWarpCombineSplits;
    const long rows = static_cast<long>(B) * Hq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = warp_combine ? dim3(static_cast<unsigned>((rows + kDecodeWarpCombineThreads / 32 - 1) /
                                                            (kDecodeWarpCombineThreads / 32)))
                               : dim3(static_cast<unsigned>(B) * static_cast<unsigned>(Hq));
    cfg.blockDim = dim3(warp_combine ? kDecodeWarpCombineThreads : kCombineThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, warp_combine ? decode_combine_warp_kernel<D> : decode_combine_kernel<D>,
                                             static_cast<const float*>(o_part), static_cast<const float*>(lse_part),
                                             seqlens, o_f32 ? nullptr : static_cast<__nv_bfloat16*>(o),
                                             o_f32 ? static_cast<float*>(o) : nullptr, lse, B, Hq, Smax, num_splits);
    if (e != cudaSuccess) return cuda_failure("decode combine launch", cudaGetErrorString(e));
    return launch_status(warp_combine ? "decode_combine_warp_kernel" : "decode_combine_kernel");
}

// Workspace of a padded forward: q, k, v and o at Dp, then the inner call's own workspace.
struct PadFwd {
    size_t q_off, k_off, v_off, o_off, inner_off, total;
    int Dp;
};

PadFwd pad_fwd_workspace(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype, float rope_base,
                         int q_pos0) {
    PadFwd w{};
    w.Dp = padded_dim(D);
    const size_t es_in = dtype == ATTN_FP32 ? 4 : 2, es_out = dtype == ATTN_BF16 ? 2 : 4;
    const size_t qe = static_cast<size_t>(B) * Sq * Hq * w.Dp, ke = static_cast<size_t>(B) * Skv * Hkv * w.Dp;
    w.q_off = 0;
    w.k_off = round_up(qe * es_in, 256);
    w.v_off = round_up(w.k_off + ke * es_in, 256);
    w.o_off = round_up(w.v_off + ke * es_in, 256);
    w.inner_off = round_up(w.o_off + qe * es_out, 256);
    w.total = w.inner_off + ex_workspace(B, Hq, Hkv, Sq, Skv, w.Dp, dtype, rope_base > 0.f, q_pos0).total;
    return w;
}

attn_status fwd_padded(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int Sq, int Skv, int D, float scale, int causal, attn_dtype dtype, float rope_base, int q_pos0,
                       void* workspace, size_t workspace_bytes, cudaStream_t st, MaskArg mk = MaskArg{}) {
    attn_status s = check_common(B, Hq, Hkv, Sq, Skv, 64, scale, causal);   // everything but D
    if (s != ATTN_OK) return s;
    if (!paddable_dim(D)) return ATTN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP32 && dtype != ATTN_BF16_OUT_F32) return ATTN_ERR_INVALID_ARG;
    const PadFwd w = pad_fwd_workspace(B, Hq, Hkv, Sq, Skv, D, dtype, rope_base, q_pos0);
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return ATTN_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int es_in = dtype == ATTN_FP32 ? 4 : 2, es_out = dtype == ATTN_BF16 ? 2 : 4;
    const long qrows = static_cast<long>(B) * Sq * Hq, krows = static_cast<long>(B) * Skv * Hkv;
    if ((s = launch_pad(q, ws + w.q_off, qrows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    if ((s = launch_pad(k, ws + w.k_off, krows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    if ((s = launch_pad(v, ws + w.v_off, krows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    s = fwd_impl(ws + w.q_off, ws + w.k_off, ws + w.v_off, ws + w.o_off, lse, B, Hq, Hkv, Sq, Skv, w.Dp, scale,
                 causal, dtype, rope_base, q_pos0, ws + w.inner_off, w.total - w.inner_off, st, D, mk);
    if (s != ATTN_OK) return s;
    return launch_pad(ws + w.o_off, o, qrows, w.Dp * es_out, D * es_out, true, st);
}

// Layout of the attn_bwd workspace: rope table (with RoPE), fp32 copies of rotated q, dO,
// rotated k, v, then D_i = dO . O per row.
struct BwdWorkspace {
    size_t tab_off, q_off, do_off, k_off, v_off, d_off, total;
    int positions;
};

BwdWorkspace bwd_workspace(int B, int Hq, int Hkv, int Sq, int Skv, int D, bool rope, int q_pos0) {
    BwdWorkspace w{};
    const long pq = static_cast<long>(q_pos0) + Sq;
    w.positions = rope ? static_cast<int>(pq > Skv ? pq : Skv) : 0;
    const size_t tab = static_cast<size_t>(w.positions) * (D / 2) * sizeof(float2);
    const size_t qb = static_cast<size_t>(B) * Sq * Hq * D * sizeof(float);
    const size_t kb = static_cast<size_t>(B) * Skv * Hkv * D * sizeof(float);
    w.tab_off = 0;
    w.q_off = round_up(tab, 256);
    w.do_off = round_up(w.q_off + qb, 256);
    w.k_off = round_up(w.do_off + qb, 256);
    w.v_off = round_up(w.k_off + kb, 256);
    w.d_off = round_up(w.v_off + kb, 256);
    w.total = round_up(w.d_off + static_cast<size_t>(B) * Hq * Sq * sizeof(float), 256);
    return w;
}

template <int D, typename T>
attn_status launch_bwd(const T* q, const T* k, const T* v, const T* o, const float* lse, const T* dout, void* dq,
                       void* dk, void* dv, bool g_f32, int B, int Hq, int Hkv, int Sq, int Skv, float scale,
                       int causal, const float2* tab, int q_pos0, uint8_t* ws, const BwdWorkspace& w,
                       cudaStream_t st, MaskArg mk) {
    float* Qf = reinterpret_cast<float*>(ws + w.q_off);
    float* dOf = reinterpret_cast<float*>(ws + w.do_off);
    float* Kf = reinterpret_cast<float*>(ws + w.k_off);
    float* Vf = reinterpret_cast<float*>(ws + w.v_off);
    float* Dvec = reinterpret_cast<float*>(ws + w.d_off);
    const long nq = static_cast<long>(B) * Sq * Hq, nk = static_cast<long>(B) * Skv * Hkv;
    bwd_prep_q_kernel<T><<<static_cast<unsigned>((nq * 32 + 255) / 256), 256, 0, st>>>(q, o, dout, Qf, dOf, Dvec, tab,
                                                                                      nq, Sq, Hq, D, q_pos0);
    attn_status s = launch_status("bwd_prep_q_kernel");
    if (s != ATTN_OK) return s;
    bwd_prep_kv_kernel<T><<<static_cast<unsigned>((nk * 32 + 255) / 256), 256, 0, st>>>(k, v, Kf, Vf, tab, nk, Skv,
                                                                                       Hkv, D);
    if ((s = launch_status("bwd_prep_kv_kernel")) != ATTN_OK) return s;
    BwdParams p{};
    p.Qf = Qf;
    p.Kf = Kf;
    p.Vf = Vf;
    p.dOf = dOf;
    p.lse = lse;
    p.Dvec = Dvec;
    p.tab = tab;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sq = Sq;
    p.Skv = Skv;
    p.q_pos0 = q_pos0;
    p.causal = causal;
    p.scale = scale;
    p.mask = mk.ptr;
    p.mask_bs = mk.bs;
    p.mask_hs = mk.hs;
    const size_t smem_dq = 2 * kBwdTile * D * sizeof(float);
    const size_t smem_dkdv = (2 * kBwdTile * D + 2 * kBwdTile) * sizeof(float);
    if ((s = prepare_kernel(reinterpret_cast<const void*>(bwd_dq_kernel<D>), static_cast<int>(smem_dq),
                            "cudaFuncSetAttribute(bwd_dq_kernel)")) != ATTN_OK)
        return s;
    if ((s = prepare_kernel(reinterpret_cast<const void*>(bwd_dkdv_kernel<D>), static_cast<int>(smem_dkdv),
                            "cudaFuncSetAttribute(bwd_dkdv_kernel)")) != ATTN_OK)
        return s;
    p.g_f32 = g_f32 ? static_cast<float*>(dq) : nullptr;
    p.g_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dq);
    bwd_dq_kernel<D><<<dim3((Sq + kBwdRows - 1) / kBwdRows, Hq, B), kBwdThreads, smem_dq, st>>>(p);
    if ((s = launch_status("bwd_dq_kernel")) != ATTN_OK) return s;
    p.g_f32 = g_f32 ? static_cast<float*>(dk) : nullptr;
    p.g_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dk);
    bwd_dkdv_kernel<D><<<dim3((Skv + kBwdRows - 1) / kBwdRows, Hkv, B), kBwdThreads, smem_dkdv, st>>>(
        p, g_f32 ? static_cast<float*>(dv) : nullptr, g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dv));
    return launch_status("bwd_dkdv_kernel");
}

// Layout of the bf16 (tensor-core) attn_bwd workspace: rope table, D_i, and with RoPE the
// rotated q and k as hi/lo bf16 pairs.
struct BmWorkspace {
    size_t tab_off, d_off, l2_off, qh_off, ql_off, kh_off, kl_off, total;
    int positions;
};

BmWorkspace bm_workspace(int B, int Hq, int Hkv, int Sq, int Skv, int D, bool rope, int q_pos0) {
    BmWorkspace w{};
    const long pq = static_cast<long>(q_pos0) + Sq;
    w.positions = rope ? static_cast<int>(pq > Skv ? pq : Skv) : 0;
    const size_t tab = static_cast<size_t>(w.positions) * (D / 2) * sizeof(float2);
    const size_t qb = rope ? static_cast<size_t>(B) * Sq * Hq * D * 2 : 0;
    const size_t kb = rope ? static_cast<size_t>(B) * Skv * Hkv * D * 2 : 0;
    w.tab_off = 0;
    w.d_off = round_up(tab, 256);
    w.l2_off = round_up(w.d_off + static_cast<size_t>(B) * Hq * Sq * sizeof(float), 256);
    w.qh_off = round_up(w.l2_off + static_cast<size_t>(B) * Hq * Sq * sizeof(float), 256);
    w.ql_off = round_up(w.qh_off + qb, 256);
    w.kh_off = round_up(w.ql_off + qb, 256);
    w.kl_off = round_up(w.kh_off + kb, 256);
    w.total = round_up(w.kl_off + kb, 256);
    return w;
}

// The tensor-core (tcgen05) backward for unmasked bf16 problems whose query length is a multiple
// of 4 (the per-row LSE and D arrays are read as 2-D TMA rows); the mma.sync kernels cover the rest.
bool bwd_tc_eligible(int Sq, const MaskArg& mk) { return mk.ptr == nullptr && Sq % 4 == 0; }

template <int D, bool ROPE>
attn_status launch_bwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                          const __nv_bfloat16* o, const float* lse, const __nv_bfloat16* dout, void* dq, void* dk,
                          void* dv, bool g_f32, int B, int Hq, int Hkv, int Sq, int Skv, float scale, int causal,
                          const float2* tab, int q_pos0, uint8_t* ws, const BmWorkspace& w, cudaStream_t st) {
    float* Dvec = reinterpret_cast<float*>(ws + w.d_off);
    float* lse2 = reinterpret_cast<float*>(ws + w.l2_off);
    const long nq = static_cast<long>(B) * Sq * Hq;
    bwd_rowdot_kernel<D><<<static_cast<unsigned>((nq * (D / 8) + 255) / 256), 256, 0, st>>>(o, dout, Dvec, nq, Sq, Hq,
                                                                                       lse, lse2);
    attn_status s = launch_status("bwd_rowdot_kernel");
    if (s != ATTN_OK) return s;
    const __nv_bfloat16 *qh = q, *ql = q, *kh = k, *kl = k;
    if (ROPE) {
        uint32_t* pqh = reinterpret_cast<uint32_t*>(ws + w.qh_off);
        uint32_t* pql = reinterpret_cast<uint32_t*>(ws + w.ql_off);
        uint32_t* pkh = reinterpret_cast<uint32_t*>(ws + w.kh_off);
        uint32_t* pkl = reinterpret_cast<uint32_t*>(ws + w.kl_off);
        const long nqp = nq * (D / 2), nkp = static_cast<long>(B) * Skv * Hkv * (D / 2);
        bwd_rope_split_kernel<<<static_cast<unsigned>(min((nqp + 255) / 256, 148L * 64)), 256, 0, st>>>(
            reinterpret_cast<const uint32_t*>(q), pqh, pql, tab, nqp, Sq, Hq, D, q_pos0);
        if ((s = launch_status("bwd_rope_split_kernel(q)")) != ATTN_OK) return s;
        bwd_rope_split_kernel<<<static_cast<unsigned>(min((nkp + 255) / 256, 148L * 64)), 256, 0, st>>>(
            reinterpret_cast<const uint32_t*>(k), pkh, pkl, tab, nkp, Skv, Hkv, D, 0);
        if ((s = launch_status("bwd_rope_split_kernel(k)")) != ATTN_OK) return s;
        qh = reinterpret_cast<const __nv_bfloat16*>(pqh);
        ql = reinterpret_cast<const __nv_bfloat16*>(pql);
        kh = reinterpret_cast<const __nv_bfloat16*>(pkh);
        kl = reinterpret_cast<const __nv_bfloat16*>(pkl);
    }
    CUtensorMap tq, tql, tk, tkl, tv, tdo, tl2, tdv;
    if (!make_tmap_bshd(&tq, qh, B, Sq, Hq, D) || !make_tmap_bshd(&tql, ql, B, Sq, Hq, D) ||
        !make_tmap_bshd(&tk, kh, B, Skv, Hkv, D) || !make_tmap_bshd(&tkl, kl, B, Skv, Hkv, D) ||
        !make_tmap_bshd(&tv, v, B, Skv, Hkv, D) || !make_tmap_bshd(&tdo, dout, B, Sq, Hq, D) ||
        !make_tmap_rows_f32(&tl2, lse2, static_cast<long>(B) * Hq, Sq) ||
        !make_tmap_rows_f32(&tdv, Dvec, static_cast<long>(B) * Hq, Sq))
        return ATTN_ERR_CUDA;
    using C = BtCfg<D, ROPE>;
    BtParams p{};
    p.lse2 = lse2;
    p.Dvec = Dvec;
    p.tab = tab;
    p.B = B, p.Hq = Hq, p.Hkv = Hkv, p.Sq = Sq, p.Skv = Skv, p.q_pos0 = q_pos0, p.causal = causal;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    auto kdq = bwd_dq_tc_kernel<D, ROPE>;
    auto kkv = bwd_dkdv_tc_kernel<D, ROPE>;
    if ((s = prepare_kernel(reinterpret_cast<const void*>(kdq), C::SMEM_Q, "bwd_dq_tc_kernel set-up", kBtLaunchRegsMin)) != ATTN_OK)
        return s;
    if ((s = prepare_kernel(reinterpret_cast<const void*>(kkv), C::SMEM_K, "bwd_dkdv_tc_kernel set-up", kBtKvLaunchRegsMin)) != ATTN_OK)
        return s;
    const long grid_q = static_cast<long>((Sq + 127) / 128) * B * Hq;
    const long grid_k = static_cast<long>((Skv + 127) / 128) * B * Hkv;
    if (grid_q > 2147483647L || grid_k > 2147483647L) return ATTN_ERR_UNSUPPORTED;
    p.g_f32 = g_f32 ? static_cast<float*>(dq) : nullptr;
    p.g_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dq);
    kdq<<<static_cast<unsigned>(grid_q), kBtThreads, C::SMEM_Q, st>>>(tq, tql, tk, tkl, tv, tdo, p);
    if ((s = launch_status("bwd_dq_tc_kernel")) != ATTN_OK) return s;
    p.g_f32 = g_f32 ? static_cast<float*>(dk) : nullptr;
    p.g_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dk);
    p.g2_f32 = g_f32 ? static_cast<float*>(dv) : nullptr;
    p.g2_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dv);
    kkv<<<static_cast<unsigned>(grid_k), kBtKvThreads, C::SMEM_K, st>>>(tq, tql, tk, tkl, tv, tdo, tl2, tdv, p);
    return launch_status("bwd_dkdv_tc_kernel");
}

template <int D, bool ROPE>
attn_status launch_bwd_mma(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                           const __nv_bfloat16* o, const float* lse, const __nv_bfloat16* dout, void* dq, void* dk,
                           void* dv, bool g_f32, int B, int Hq, int Hkv, int Sq, int Skv, float scale, int causal,
                           const float2* tab, int q_pos0, uint8_t* ws, const BmWorkspace& w, cudaStream_t st,
                           MaskArg mk) {
    float* Dvec = reinterpret_cast<float*>(ws + w.d_off);
    const long nq = static_cast<long>(B) * Sq * Hq;
    bwd_rowdot_kernel<D><<<static_cast<unsigned>((nq * (D / 8) + 255) / 256), 256, 0, st>>>(o, dout, Dvec, nq, Sq, Hq);
    attn_status s = launch_status("bwd_rowdot_kernel");
    if (s != ATTN_OK) return s;
    BmParams p{};
    p.q = q;
    p.k = k;
    if (ROPE) {
        uint32_t* qh = reinterpret_cast<uint32_t*>(ws + w.qh_off);
        uint32_t* ql = reinterpret_cast<uint32_t*>(ws + w.ql_off);
        uint32_t* kh = reinterpret_cast<uint32_t*>(ws + w.kh_off);
        uint32_t* kl = reinterpret_cast<uint32_t*>(ws + w.kl_off);
        const long nqp = nq * (D / 2), nkp = static_cast<long>(B) * Skv * Hkv * (D / 2);
        bwd_rope_split_kernel<<<static_cast<unsigned>(min((nqp + 255) / 256, 148L * 64)), 256, 0, st>>>(
            reinterpret_cast<const uint32_t*>(q), qh, ql, tab, nqp, Sq, Hq, D, q_pos0);
        if ((s = launch_status("bwd_rope_split_kernel(q)")) != ATTN_OK) return s;
        bwd_rope_split_kernel<<<static_cast<unsigned>(min((nkp + 255) / 256, 148L * 64)), 256, 0, st>>>(
            reinterpret_cast<const uint32_t*>(k), kh, kl, tab, nkp, Skv, Hkv, D, 0);
        if ((s = launch_status("bwd_rope_split_kernel(k)")) != ATTN_OK) return s;
        p.q = reinterpret_cast<const __nv_bfloat16*>(qh);
        p.ql = reinterpret_cast<const __nv_bfloat16*>(ql);
        p.k = reinterpret_cast<const __nv_bfloat16*>(kh);
        p.kl = reinterpret_cast<const __nv_bfloat16*>(kl);
    }
    p.v = v;
    p.dout = dout;
    p.lse = lse;
    p.Dvec = Dvec;
    p.tab = tab;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Sq = Sq;
    p.Skv = Skv;
    p.q_pos0 = q_pos0;
    p.causal = causal;
    p.scale = scale;
    p.mask = mk.ptr;
    p.mask_bs = mk.bs;
    p.mask_hs = mk.hs;
    using C = BmCfg<D, ROPE>;
    const bool masked = mk.ptr != nullptr;   // separate instantiations: the unmasked ones carry no mask code
    auto kdq = masked ? bwd_dq_mma_kernel<D, ROPE, true> : bwd_dq_mma_kernel<D, ROPE, false>;
    auto kkv = masked ? bwd_dkdv_mma_kernel<D, ROPE, true> : bwd_dkdv_mma_kernel<D, ROPE, false>;
    if ((s = prepare_kernel(reinterpret_cast<const void*>(kdq), C::SMEM, "cudaFuncSetAttribute(bwd_dq_mma_kernel)")) !=
        ATTN_OK)
        return s;
    if ((s = prepare_kernel(reinterpret_cast<const void*>(kkv), C::SMEM,
                            "cudaFuncSetAttribute(bwd_dkdv_mma_kernel)")) != ATTN_OK)
        return s;
    p.g_f32 = g_f32 ? static_cast<float*>(dq) : nullptr;
    p.g_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dq);
    kdq<<<dim3((Sq + kBmRows - 1) / kBmRows, Hq, B), kBmThreads, C::SMEM, st>>>(p);
    if ((s = launch_status("bwd_dq_mma_kernel")) != ATTN_OK) return s;
    p.g_f32 = g_f32 ? static_cast<float*>(dk) : nullptr;
    p.g_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dk);
    p.g2_f32 = g_f32 ? static_cast<float*>(dv) : nullptr;
    p.g2_bf16 = g_f32 ? nullptr : static_cast<__nv_bfloat16*>(dv);
    kkv<<<dim3((Skv + kBmRows - 1) / kBmRows, Hkv, B), kBmThreads, C::SMEM, st>>>(p);
    return launch_status("bwd_dkdv_mma_kernel");
}

}  // namespace

namespace {

size_t bwd_inner_bytes(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype, float rope_base, int q_pos0) {
    if (dtype == ATTN_FP32) return bwd_workspace(B, Hq, Hkv, Sq, Skv, D, rope_base > 0.f, q_pos0).total;
    return bm_workspace(B, Hq, Hkv, Sq, Skv, D, rope_base > 0.f, q_pos0).total;
}

// Workspace of a padded backward: q, k, v, o, dout and dq, dk, dv at Dp, then the inner call's.
struct PadBwd {
    size_t q_off, k_off, v_off, o_off, g_off, dq_off, dk_off, dv_off, inner_off, total;
    int Dp;
};

PadBwd pad_bwd_workspace(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype, float rope_base,
                         int q_pos0) {
    PadBwd w{};
    w.Dp = padded_dim(D);
    const size_t es_in = dtype == ATTN_FP32 ? 4 : 2, es_g = dtype == ATTN_BF16 ? 2 : 4;
    const size_t qe = static_cast<size_t>(B) * Sq * Hq * w.Dp, ke = static_cast<size_t>(B) * Skv * Hkv * w.Dp;
    w.q_off = 0;
    w.k_off = round_up(qe * es_in, 256);
    w.v_off = round_up(w.k_off + ke * es_in, 256);
    w.o_off = round_up(w.v_off + ke * es_in, 256);
    w.g_off = round_up(w.o_off + qe * es_in, 256);
    w.dq_off = round_up(w.g_off + qe * es_in, 256);
    w.dk_off = round_up(w.dq_off + qe * es_g, 256);
    w.dv_off = round_up(w.dk_off + ke * es_g, 256);
    w.inner_off = round_up(w.dv_off + ke * es_g, 256);
    w.total = w.inner_off + bwd_inner_bytes(B, Hq, Hkv, Sq, Skv, w.Dp, dtype, rope_base, q_pos0);
    return w;
}

attn_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                     int causal, attn_dtype dtype, float rope_base, int q_pos0, void* workspace,
                     size_t workspace_bytes, attn_stream_t stream, int rope_dim, MaskArg mk);

}  // namespace

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype, float rope_base,
                               int q_pos0) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || D <= 0 || q_pos0 < 0) return 0;
    if (!native_dim(D)) return paddable_dim(D) ? pad_bwd_workspace(B, Hq, Hkv, Sq, Skv, D, dtype, rope_base, q_pos0).total : 0;
    return bwd_inner_bytes(B, Hq, Hkv, Sq, Skv, D, dtype, rope_base, q_pos0);
}

namespace {

// attn_bwd and attn_bwd_masked: native head dims go straight to bwd_impl, others through padding.
attn_status bwd_entry(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                      void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                      int causal, attn_dtype dtype, float rope_base, int q_pos0, void* workspace,
                      size_t workspace_bytes, attn_stream_t stream, MaskArg mk) {
    if (D <= 0 || native_dim(D))
        return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, rope_base,
                        q_pos0, workspace, workspace_bytes, stream, D, mk);
    attn_status s = check_common(B, Hq, Hkv, Sq, Skv, 64, scale, causal);   // everything but D
    if (s != ATTN_OK) return s;
    if (!paddable_dim(D)) return ATTN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP32 && dtype != ATTN_BF16_OUT_F32) return ATTN_ERR_INVALID_ARG;
    const PadBwd w = pad_bwd_workspace(B, Hq, Hkv, Sq, Skv, D, dtype, rope_base, q_pos0);
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return ATTN_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int es_in = dtype == ATTN_FP32 ? 4 : 2, es_g = dtype == ATTN_BF16 ? 2 : 4;
    const long qrows = static_cast<long>(B) * Sq * Hq, krows = static_cast<long>(B) * Skv * Hkv;
    if ((s = launch_pad(q, ws + w.q_off, qrows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    if ((s = launch_pad(k, ws + w.k_off, krows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    if ((s = launch_pad(v, ws + w.v_off, krows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    if ((s = launch_pad(o, ws + w.o_off, qrows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    if ((s = launch_pad(dout, ws + w.g_off, qrows, D * es_in, w.Dp * es_in, false, st)) != ATTN_OK) return s;
    s = bwd_impl(ws + w.q_off, ws + w.k_off, ws + w.v_off, ws + w.o_off, lse, ws + w.g_off, ws + w.dq_off,
                 ws + w.dk_off, ws + w.dv_off, B, Hq, Hkv, Sq, Skv, w.Dp, scale, causal, dtype, rope_base, q_pos0,
                 ws + w.inner_off, w.total - w.inner_off, stream, D, mk);
    if (s != ATTN_OK) return s;
    if ((s = launch_pad(ws + w.dq_off, dq, qrows, w.Dp * es_g, D * es_g, true, st)) != ATTN_OK) return s;
    if ((s = launch_pad(ws + w.dk_off, dk, krows, w.Dp * es_g, D * es_g, true, st)) != ATTN_OK) return s;
    return launch_pad(ws + w.dv_off, dv, krows, w.Dp * es_g, D * es_g, true, st);
}

}  // namespace

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                     int causal, attn_dtype dtype, float rope_base, int q_pos0, void* workspace,
                     size_t workspace_bytes, attn_stream_t stream) {
    return bwd_entry(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, rope_base,
                     q_pos0, workspace, workspace_bytes, stream, MaskArg{});
}

attn_status attn_bwd_masked(const void* q, const void* k, const void* v, const float* mask, int64_t mask_batch_stride,
                            int64_t mask_head_stride, const void* o, const float* lse, const void* dout, void* dq,
                            void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale, int causal,
                            attn_dtype dtype, float rope_base, int q_pos0, void* workspace, size_t workspace_bytes,
                            attn_stream_t stream) {
    if (!mask || (reinterpret_cast<uintptr_t>(mask) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if (mask_batch_stride < 0 || mask_head_stride < 0) return ATTN_ERR_INVALID_ARG;
    MaskArg mk;
    mk.ptr = mask;
    mk.bs = static_cast<long>(mask_batch_stride);
    mk.hs = static_cast<long>(mask_head_stride);
    return bwd_entry(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, rope_base,
                     q_pos0, workspace, workspace_bytes, stream, mk);
}

namespace {

attn_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                     int causal, attn_dtype dtype, float rope_base, int q_pos0, void* workspace,
                     size_t workspace_bytes, attn_stream_t stream, int rope_dim, MaskArg mk) {
    attn_status s = check_common(B, Hq, Hkv, Sq, Skv, D, scale, causal);
    if (s != ATTN_OK) return s;
    if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP32 && dtype != ATTN_BF16_OUT_F32) return ATTN_ERR_INVALID_ARG;
    const bool rope = rope_base > 0.f;
    if (rope && !isfinite(rope_base)) return ATTN_ERR_INVALID_ARG;
    if (q_pos0 < 0) return ATTN_ERR_INVALID_ARG;
    if (Hq > 65535 || B > 65535 || Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
    const BwdWorkspace w = bwd_workspace(B, Hq, Hkv, Sq, Skv, D, rope, q_pos0);
    const BmWorkspace wm = bm_workspace(B, Hq, Hkv, Sq, Skv, D, rope, q_pos0);
    const size_t need = dtype == ATTN_FP32 ? w.total : wm.total;
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return ATTN_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const float2* tab = nullptr;
    if (rope) {
        float2* t = reinterpret_cast<float2*>(ws + w.tab_off);   // offset 0 in both layouts
        const long n = static_cast<long>(w.positions) * (D / 2);
        rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0, st>>>(
            t, w.positions, D, static_cast<double>(rope_base), rope_dim);
        if ((s = launch_status("rope_table_kernel")) != ATTN_OK) return s;
        tab = t;
    }
    const bool g_f32 = dtype != ATTN_BF16;
    if (dtype == ATTN_FP32) {
        const float *qf = static_cast<const float*>(q), *kf = static_cast<const float*>(k),
                    *vf = static_cast<const float*>(v), *of = static_cast<const float*>(o),
                    *gf = static_cast<const float*>(dout);
        return D == 64 ? launch_bwd<64>(qf, kf, vf, of, lse, gf, dq, dk, dv, true, B, Hq, Hkv, Sq, Skv, scale, causal,
                                        tab, q_pos0, ws, w, st, mk)
                       : launch_bwd<128>(qf, kf, vf, of, lse, gf, dq, dk, dv, true, B, Hq, Hkv, Sq, Skv, scale,
                                         causal, tab, q_pos0, ws, w, st, mk);
    }
    using bf = __nv_bfloat16;
    const bf *qb = static_cast<const bf*>(q), *kb = static_cast<const bf*>(k), *vb = static_cast<const bf*>(v),
             *ob = static_cast<const bf*>(o), *gb = static_cast<const bf*>(dout);
    if (bwd_tc_eligible(Sq, mk)) {
        if (D == 64)
            return rope ? launch_bwd_tc<64, true>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv, scale,
                                                  causal, tab, q_pos0, ws, wm, st)
                        : launch_bwd_tc<64, false>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv,
                                                   scale, causal, tab, q_pos0, ws, wm, st);
        return rope ? launch_bwd_tc<128, true>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv, scale,
                                               causal, tab, q_pos0, ws, wm, st)
                    : launch_bwd_tc<128, false>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv, scale,
                                                causal, tab, q_pos0, ws, wm, st);
    }
    if (D == 64)
        return rope ? launch_bwd_mma<64, true>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv, scale,
                                               causal, tab, q_pos0, ws, wm, st, mk)
                    : launch_bwd_mma<64, false>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv, scale,
                                                causal, tab, q_pos0, ws, wm, st, mk);
    return rope ? launch_bwd_mma<128, true>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv, scale,
                                            causal, tab, q_pos0, ws, wm, st, mk)
                : launch_bwd_mma<128, false>(qb, kb, vb, ob, lse, gb, dq, dk, dv, g_f32, B, Hq, Hkv, Sq, Skv, scale,
                                             causal, tab, q_pos0, ws, wm, st, mk);
}

// Argument rules of the split-KV decode, shared by attn_decode and attn_decode_noalloc so that the
// two entry points accept exactly the same calls (they differ only in where the partials live).
attn_status decode_check(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens, const void* o,
                         int B, int Hq, int Hkv, int Smax, int D, float scale, int num_splits, attn_dtype dtype) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || num_splits <= 0) return ATTN_ERR_INVALID_ARG;
    if (Smax == 0) return ATTN_ERR_EMPTY_KV;
    if (Smax < 0) return ATTN_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ATTN_ERR_DIM_MISMATCH;
    if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (!q || !kcache || !vcache || !seqlens || !o) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_BF16_OUT_F32)
        return dtype == ATTN_FP32 ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    if (num_splits > 65535) return ATTN_ERR_UNSUPPORTED;
    if (static_cast<long>(B) * Hq > 2147483647L) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

// Launch of a checked decode with its partials at `part` (attn_decode_workspace_size bytes, 16-byte
// aligned): o_part [B*Hq*num_splits][D] fp32, then lse_part [B*Hq*num_splits] fp32.
attn_status decode_launch(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens, void* o,
                          float* lse, int B, int Hq, int Hkv, int Smax, int D, float scale, int num_splits, void* part,
                          attn_dtype dtype, cudaStream_t st) {
    const size_t slots = static_cast<size_t>(B) * Hq * num_splits;
    float* o_part = static_cast<float*>(part);
    float* lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(part) + round_up(slots * D * sizeof(float), 256));
    const bool o_f32 = dtype == ATTN_BF16_OUT_F32;
    if (D == 64)
        return launch_decode<64>(q, kcache, vcache, seqlens, o, o_f32, lse, B, Hq, Hkv, Smax, scale, num_splits, o_part,
                                 lse_part, st);
    return launch_decode<128>(q, kcache, vcache, seqlens, o, o_f32, lse, B, Hq, Hkv, Smax, scale, num_splits, o_part,
                              lse_part, st);
}

}  // namespace

// ------------------------------------------------------------------------------------------
// Built-in decode scratch for callers that cannot allocate device memory.
//
// attn_decode needs somewhere to put the per-split partial outputs; normally the caller passes a
// workspace.  Some callers cannot provide one: code that runs inside a host framework owning
// every device allocation (a plugin handed only its input and output buffers), or a serving
// path that must not call cudaMalloc because it can synchronise the device and take an
// unbounded time.  For them attn_decode_noalloc keeps the partials in this fixed array, which
// exists once per GPU that loads the library and stays allocated until the process exits.
// ------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};   // device address of g_noalloc_scratch, per device

// Device address of the scratch array on the current device, looked up once per device.  A
// host-side reference to g_noalloc_scratch is only a stand-in for the symbol, never a device
// address, so the address must come from cudaGetSymbolAddress with that device current.
attn_status noalloc_scratch(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_failure("cudaGetDevice", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return cuda_failure("attn_decode_noalloc", "device ordinal out of range");
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr)
            return cuda_failure("cudaGetSymbolAddress(g_noalloc_scratch)",
                                e != cudaSuccess ? cudaGetErrorString(e) : "null address");
        g_noalloc_addr[dev] = ptr;
    }
    *out = g_noalloc_addr[dev];
    return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Sq,
                     int Skv, int D, float scale, int causal, attn_dtype dtype, attn_stream_t stream) {
    if (D > 0 && !native_dim(D)) {
        // other head dims pad through a workspace: attn_fwd_ex
        snprintf(g_last_error, sizeof(g_last_error), "head dim %d needs attn_fwd_ex with a workspace", D);
        return ATTN_ERR_UNSUPPORTED;
    }
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, 0.f, 0, nullptr, 0,
                    static_cast<cudaStream_t>(stream), D);
}

attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                        int Sq, int Skv, int D, float scale, int causal, attn_dtype dtype, float rope_base, int q_pos0,
                        void* workspace, size_t workspace_bytes, attn_stream_t stream) {
    if (D > 0 && !native_dim(D))
        return fwd_padded(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, rope_base, q_pos0, workspace,
                          workspace_bytes, static_cast<cudaStream_t>(stream));
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, rope_base, q_pos0, workspace,
                    workspace_bytes, static_cast<cudaStream_t>(stream), D);
}

attn_status attn_fwd_masked(const void* q, const void* k, const void* v, const float* mask, int64_t mask_batch_stride,
                            int64_t mask_head_stride, void* o, float* lse, int B, int Hq, int Hkv, int Sq, int Skv,
                            int D, float scale, int causal, attn_dtype dtype, float rope_base, int q_pos0,
                            void* workspace, size_t workspace_bytes, attn_stream_t stream) {
    if (!mask || (reinterpret_cast<uintptr_t>(mask) & 3u) != 0) return ATTN_ERR_INVALID_ARG;
    if (mask_batch_stride < 0 || mask_head_stride < 0) return ATTN_ERR_INVALID_ARG;
    MaskArg mk;
    mk.ptr = mask;
    mk.bs = static_cast<long>(mask_batch_stride);
    mk.hs = static_cast<long>(mask_head_stride);
    if (D > 0 && !native_dim(D))
        return fwd_padded(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, rope_base, q_pos0, workspace,
                          workspace_bytes, static_cast<cudaStream_t>(stream), mk);
    return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, dtype, rope_base, q_pos0, workspace,
                    workspace_bytes, static_cast<cudaStream_t>(stream), D, mk);
}

size_t attn_fwd_ex_workspace_size(int B, int Hq, int Hkv, int Sq, int Skv, int D, attn_dtype dtype, float rope_base,
                                  int q_pos0) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || D <= 0 || q_pos0 < 0) return 0;
    if (!native_dim(D)) return paddable_dim(D) ? pad_fwd_workspace(B, Hq, Hkv, Sq, Skv, D, dtype, rope_base, q_pos0).total : 0;
    return ex_workspace(B, Hq, Hkv, Sq, Skv, D, dtype, rope_base > 0.f, q_pos0).total;
}

int attn_fwd_kv_splits(int B, int Hq, int Sq, int Skv, attn_dtype dtype) {
    if (B <= 0 || Hq <= 0 || Sq <= 0 || Skv <= 0) return 1;
    return fwd_kv_splits(B, Hq, Sq, Skv, dtype);
}

size_t attn_decode_workspace_size(int B, int Hq, int D, int num_splits) {
    if (B <= 0 || Hq <= 0 || D <= 0 || num_splits <= 0) return 0;
    const size_t slots = static_cast<size_t>(B) * Hq * num_splits;
    return round_up(slots * D * sizeof(float), 256) + round_up(slots * sizeof(float), 256);
}

attn_status attn_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens, void* o,
                        float* lse, int B, int Hq, int Hkv, int Smax, int D, float scale, int num_splits,
                        void* workspace, size_t workspace_bytes, attn_dtype dtype, attn_stream_t stream) {
    const attn_status s = decode_check(q, kcache, vcache, seqlens, o, B, Hq, Hkv, Smax, D, scale, num_splits, dtype);
    if (s != ATTN_OK) return s;
    const size_t need = attn_decode_workspace_size(B, Hq, D, num_splits);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return ATTN_ERR_WORKSPACE;
    return decode_launch(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Smax, D, scale, num_splits, workspace, dtype,
                         static_cast<cudaStream_t>(stream));
}

attn_status attn_decode_noalloc(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                                void* o, float* lse, int B, int Hq, int Hkv, int Smax, int D, float scale,
                                int num_splits, attn_dtype dtype, attn_stream_t stream) {
    // The same argument rules as attn_decode (one shared check), then the size check against the
    // built-in scratch in place of the caller's workspace.
    attn_status s = decode_check(q, kcache, vcache, seqlens, o, B, Hq, Hkv, Smax, D, scale, num_splits, dtype);
    if (s != ATTN_OK) return s;
    const size_t need = attn_decode_workspace_size(B, Hq, D, num_splits);
    if (need > ATTN_NOALLOC_SCRATCH_BYTES) {
        char buf[160];
        snprintf(buf, sizeof(buf), "split partials need %zu bytes, the built-in scratch holds %zu (lower num_splits or B*Hq)",
                 need, static_cast<size_t>(ATTN_NOALLOC_SCRATCH_BYTES));
        snprintf(g_last_error, sizeof(g_last_error), "attn_decode_noalloc: %s", buf);
        return ATTN_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != ATTN_OK) return s;
    // Nothing in the scratch has to start at zero: every partial the combine reads is written
    // earlier in the same call by the split kernel.
    return decode_launch(q, kcache, vcache, seqlens, o, lse, B, Hq, Hkv, Smax, D, scale, num_splits, scratch, dtype,
                         static_cast<cudaStream_t>(stream));
}

attn_status rope_apply(void* x, const int32_t* pos, int T, int H, int D, float base, attn_dtype dtype,
                       attn_stream_t stream) {
    if (T <= 0 || H <= 0 || D <= 0) return ATTN_ERR_INVALID_ARG;
    if (D % 2 != 0) return ATTN_ERR_DIM_MISMATCH;
    if (!(base > 0.f) || !isfinite(base)) return ATTN_ERR_INVALID_ARG;
    if (!x || !pos) return ATTN_ERR_INVALID_ARG;
    if (dtype != ATTN_BF16 && dtype != ATTN_FP32) return ATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & (dtype == ATTN_BF16 ? 3u : 7u)) != 0) return ATTN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = T < 65535 * 4 ? static_cast<unsigned>(T) : 65535u * 4;
    const size_t smem = (D / 2) * sizeof(float2);
    if (dtype == ATTN_BF16)
        rope_apply_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(static_cast<__nv_bfloat16*>(x), pos, T, H, D,
                                                                  static_cast<double>(base));
    else
        rope_apply_kernel<float><<<grid, 128, smem, st>>>(static_cast<float*>(x), pos, T, H, D,
                                                          static_cast<double>(base));
    return launch_status("rope_apply_kernel");
}

attn_status attn_kv_append(void* kcache, void* vcache, int32_t* seqlens, const void* k_new, const void* v_new,
                           void* q, int B, int T, int Hq, int Hkv, int Smax, int D, float rope_base,
                           attn_stream_t stream) {
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || Smax <= 0 || D <= 0) return ATTN_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ATTN_ERR_DIM_MISMATCH;
    if (D % 8 != 0) return ATTN_ERR_DIM_MISMATCH;   // value rows move as 16-byte vectors; RoPE needs D even
    if (!kcache || !vcache || !seqlens || !k_new || !v_new) return ATTN_ERR_INVALID_ARG;
    if (!isfinite(rope_base)) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(kcache) || !aligned16(vcache) || !aligned16(k_new) || !aligned16(v_new) ||
        (q != nullptr && !aligned16(q)))
        return ATTN_ERR_INVALID_ARG;
    if (B > 65535 * 32) return ATTN_ERR_UNSUPPORTED;
    kv_append_kernel<<<B, 256, (D / 2) * sizeof(float2), static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint32_t*>(kcache), static_cast<uint4*>(vcache), seqlens, static_cast<const uint32_t*>(k_new),
        static_cast<const uint4*>(v_new), static_cast<uint32_t*>(q), T, Hq, Hkv, Smax, D,
        rope_base > 0.f ? static_cast<double>(rope_base) : 0.0);
    return launch_status("kv_append_kernel");
}

attn_status attn_selftest_wait_timeout(int timeout_us, attn_stream_t stream) {
    if (timeout_us < 1 || timeout_us > 1000000) return ATTN_ERR_INVALID_ARG;
    wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(timeout_us) * 1000ull);
    return launch_status("wait_timeout_selftest_kernel");
}

const char* attn_last_error(void) { return g_last_error; }

const char* attn_status_string(attn_status s) {
    switch (s) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument";
        case ATTN_ERR_DIM_MISMATCH: return "dimension mismatch";
        case ATTN_ERR_EMPTY_KV: return "empty KV";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
        case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case ATTN_ERR_CUDA: return "CUDA error";
        case ATTN_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int attn_read_device_status(attn_stream_t stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return -1;
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return -1;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return -1;
    return v;
}

}  // extern "C"
