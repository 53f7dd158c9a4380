// Internal declarations shared by the LLA CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lla.h"

struct lla_codec {
    lla_codec_desc desc;
    int S;          // stack length fed to W_down: T*d (per-head) or T*H*d (LLA-2D)
    int device;
    // float32 copies
    float* w_up_k = nullptr;   // per-head [D][H][T][d][r_k];  2D [D][T][H][d][r_k]
    // W^K_up,t transposed with mu^K_t appended as the last row, for the query prologue:
    // per-head [D][H][T][r_k + 1][d];  2D [D][T][H][r_k + 1][d]
    float* w_up_k_t = nullptr;
    float* w_up_v = nullptr;   // per-head [D][H][T][d][r_v];  2D [D][T][H][d][r_v]
    float* mu_k = nullptr;     // per-head [D][H][S];          2D [D][S]
    float* mu_v = nullptr;
    float* bias_k = nullptr;   // b = mu W_down: per-head [D][H][r_k]; 2D [D][r_k]
    float* bias_v = nullptr;
    // bf16 W_down, transposed so that each latent dimension is one K-major row:
    // per-head [D][H][r][S]; 2D [D][r][S]
    uint16_t* w_down_k_t = nullptr;
    uint16_t* w_down_v_t = nullptr;
    // RoPE tables, filled in double precision on the host
    float* rope_cos = nullptr;  // [max_pos][d/2]
    float* rope_sin = nullptr;  // [max_pos][d/2]
    // Position features Phi_j = [cos(j theta) | sin(j theta)] as bf16, one
    // 128 x d_head tile per 128 positions, pre-arranged in the shared-memory
    // image the tensor-core decode kernel feeds to tcgen05.mma.
    uint16_t* phi_tiles = nullptr;
    int phi_num_tiles = 0;
    // bf16 copies of W_up (same layouts as w_up_k / w_up_v): the B operands of the tensor-core
    // reconstruction of a full K/V cache (lla_reconstruct_cache)
    uint16_t* w_up_k_bf16 = nullptr;
    uint16_t* w_up_v_bf16 = nullptr;
    // Device status words of the tensor-core encode (bit 2: a bounded wait gave up; word 1:
    // the first wait site that did).
    uint32_t* status = nullptr;
};

// Workspace header (first 256 bytes of every decode workspace).
struct lla_ws_header {
    uint32_t flags;      // LLA_FLAG_* bits
    uint32_t pad[63];
};

enum : uint32_t {
    LLA_FLAG_SEQ_LEN_CLAMPED = 1u,
    LLA_FLAG_POS_CLAMPED = 2u,
    LLA_FLAG_PAGE_INVALID = 4u,
    LLA_FLAG_FIT_BREAKDOWN = 8u,  // codec fit: a Cholesky pivot was not positive
};

// Where the rows of a latent store live.  Contiguous: [batch][D][max_tokens][row].  Paged: a
// pool of pages [num_pages][D][kPageTokens][row]; token j of sequence b sits in pool page
// table[b * max_pages + j / kPageTokens], slot j % kPageTokens.
constexpr int kPageTokens = 128;
struct lla_store_map {
    const int32_t* table = nullptr;  // null: contiguous
    int max_pages = 0;
    int num_pages = 0;
    // row index of (b, layer, token), or -1 when the token's page index is out of range
    __host__ __device__ long long row_index(int b, int layer, int tok, int D, int max_tokens) const {
        if (!table) return (static_cast<long long>(b) * D + layer) * max_tokens + tok;
        const int pg = table[static_cast<size_t>(b) * max_pages + tok / kPageTokens];
        if (pg < 0 || pg >= num_pages) return -1;
        return (static_cast<long long>(pg) * D + layer) * kPageTokens + tok % kPageTokens;
    }
    // tokens of sequence b usable with this map: n, cut before its first page that is out of
    // range (paged stores only)
    __device__ int usable_tokens(int b, int n) const {
        if (!table) return n;
        for (int pg = 0; pg * kPageTokens < n; ++pg) {
            const int e = table[static_cast<size_t>(b) * max_pages + pg];
            if (e < 0 || e >= num_pages) return pg * kPageTokens;
        }
        return n;
    }
};

// Common decode-call parameters after host validation.
struct lla_decode_call {
    const lla_codec* codec;
    const uint16_t* store;
    int batch, max_tokens, layer, loop;
    const float* q;
    const int32_t* q_pos;
    const int32_t* seq_lens;
    float scale;
    float* out;
    char* workspace;
    size_t workspace_bytes;
    cudaStream_t stream;
    cudaEvent_t ev_begin = nullptr;  // recorded around the main attention kernel when set
    cudaEvent_t ev_end = nullptr;
    const float* k_self = nullptr;   // optional self slot: the current token's exact loop-t
    const float* v_self = nullptr;   // key (pre-RoPE) and value, [batch][H][d_head]
    lla_store_map smap;              // paged store (max_tokens = max_pages * kPageTokens)
};

// One (layer, loop) slice of a full K/V cache rebuilt from the latent store.
struct lla_reconstruct_call {
    const lla_codec* codec;
    const uint16_t* store;
    int batch, max_tokens, layer, loop;
    const int32_t* seq_lens;
    uint16_t* k_cache;
    uint16_t* v_cache;
    long long seq_stride;
    int cache_tokens;
    cudaStream_t stream;
};
bool lla_reconstruct_tc_supported(const lla_codec* c);
lla_status lla_reconstruct_launch(const lla_reconstruct_call& rc, int impl);

// ---- bf16 helpers ---------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// ---- partial (m, l, acc[r_v]) records written by the split kernels --------
__host__ __device__ inline size_t lla_partial_floats(int r_v) { return size_t(r_v) + 2; }

// ---- host-side entry points implemented in the .cu files ------------------
size_t lla_simt_workspace_bytes(const lla_codec* c, int batch, int max_tokens);
// scratch of the CUDA-core kernel at its automatic split count (no explicit split override)
size_t lla_simt_auto_workspace_bytes(const lla_codec* c, int batch, int max_tokens);
lla_status lla_decode_simt(const lla_decode_call& call, int splits_override);
size_t lla_tc_workspace_bytes(const lla_codec* c, int batch, int max_tokens);
bool lla_tc_supported(const lla_codec* c);
lla_status lla_decode_tc(const lla_decode_call& call, int num_ctas_override);
lla_status lla_combine(const lla_decode_call& call, const float* partials, const int32_t* slot_range,
                       int splits);
// Record layout of the tensor-core kernel: persistent CTA c working on
// (part p, sequence b) writes records [(c + p*B + b)][quarter 0..3][head in part].
struct lla_tc_ranges {
    const int32_t* P;  // per-sequence tile prefix [B+1] (device)
    int G;             // CTAs of the decode launch
    int parts;         // head parts (heads per part = hc)
    int hc;
};
lla_status lla_combine_tc(const lla_decode_call& call, const float* records, const lla_tc_ranges& r);
lla_status lla_encode_launch(const lla_codec* c, const uint16_t* x, int n, int layer_begin,
                             int num_layers, const int32_t* seq_idx, const int32_t* tok_idx,
                             uint16_t* store, int batch, int max_tokens, cudaStream_t stream,
                             const lla_store_map& smap = lla_store_map());
lla_status lla_build_phi_tiles(lla_codec* c, cudaStream_t stream);
lla_status lla_encode_simt(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                           const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* store, int batch,
                           int max_tokens, cudaStream_t stream, const lla_store_map& smap);
lla_status lla_encode_tc(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                         const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* store, int batch, int max_tokens,
                         cudaStream_t stream, const lla_store_map& smap);

int lla_num_sms();
size_t lla_fit_workspace_bytes_impl(int P, int n, int S, int r);
bool lla_fit_shape_ok(int n, int S, int r);
lla_status lla_fit(int P, int n, int S, int r, const float* X, float* mu_out, float* w_out, float* sig_out, int iters,
                   void* workspace, cudaStream_t stream);
size_t lla_full_workspace_bytes(int H, int batch);
lla_status lla_full_decode(int H, float rope_base, const uint16_t* k_cache, const uint16_t* v_cache,
                           long long seq_stride, int batch, int max_tokens, const float* q, const int32_t* q_pos,
                           const int32_t* seq_lens, float scale, float* out, void* workspace, size_t workspace_bytes,
                           int num_ctas, cudaStream_t stream);

// ---- programmatic dependent launch ----------------------------------------------------------
// The kernels of one call run back to back in a stream.  A kernel launched by lla_launch with
// pdl = true is scheduled as the CTAs of the kernel before it exit (none of them triggers its
// dependents early: measured slower, the dependents then take SM resources the predecessor's
// last CTAs still need); it calls lla_grid_dependency_wait() before it touches anything that
// kernel writes (a no-op after a plain launch), so its launch and set-up overlap that kernel's
// tail.
__device__ __forceinline__ void lla_grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Asynchronous global -> shared copies of 4 or 16 bytes (no registers held while in flight);
// lla_cp_async_wait_all() waits for every copy this thread issued.
__device__ __forceinline__ void lla_cp_async4(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(uint32_t(__cvta_generic_to_shared(smem_dst))),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void lla_cp_async16(void* smem_dst, const void* gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(uint32_t(__cvta_generic_to_shared(smem_dst))),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void lla_cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t lla_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

#define LLA_CUDA_TRY(expr)                                   \
    do {                                                     \
        cudaError_t _e = (expr);                             \
        if (_e != cudaSuccess) return LLA_ERR_CUDA;          \
    } while (0)
