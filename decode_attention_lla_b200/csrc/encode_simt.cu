// CUDA-core LLA encode: c = (x - mu) W_down, written into the latent store.
//
// [LLA §3 eq. (2)]: for each token, layer, head and axis the loop stack x
// (length S = T*d_head, or T*H*d_head for LLA-2D) is projected onto r latent
// dimensions.  The kernel forms x W_down with float32 accumulation over bf16
// operands and subtracts b = mu W_down (precomputed), which equals centring
// first; the result is rounded to bf16 (nearest-even) into the store row of
// (seq_idx[i], tok_idx[i]).
//
// Tiling: one CTA per (64-token chunk, layer/head slot, axis); the K
// dimension S is walked in 64-wide slabs staged in shared memory.
#include <cuda_bf16.h>

#include "lla_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kTok = 64;
constexpr int kK = 64;
constexpr int kMaxR = 256;
constexpr int kAcc = kMaxR / (kThreads / kTok);  // 64 accumulators per thread at most

struct EncodeParams {
    const uint16_t* x;
    const int32_t* seq_idx;
    const int32_t* tok_idx;
    uint16_t* store;
    const uint16_t* wdt_k;
    const uint16_t* wdt_v;
    const float* bias_k;
    const float* bias_v;
    int n, layer_begin, num_layers, H, S, r_k, r_v, variant, batch, max_tokens, D;
    lla_store_map smap;
};

__global__ void __launch_bounds__(kThreads) encode_simt_kernel(EncodeParams p) {
    const int chunk = blockIdx.x;
    const int slot = blockIdx.y;  // L * Hg + h
    const int axis = blockIdx.z;
    const int Hg = p.variant == 0 ? p.H : 1;
    const int L = slot / Hg, h = slot - L * Hg;
    const int layer = p.layer_begin + L;
    const int r = axis == 0 ? p.r_k : p.r_v;
    const int S = p.S;
    const int tid = threadIdx.x;
    const int tok = tid % kTok, agrp = tid / kTok;  // this thread: token `tok`, latent dims agrp + 4*u

    __shared__ float xs[kTok][kK + 1];
    extern __shared__ float ws[];  // [r][kK]

    const size_t g = size_t(layer) * Hg + h;  // codec slot
    const uint16_t* W = (axis == 0 ? p.wdt_k : p.wdt_v) + g * size_t(r) * S;
    const float* bias = (axis == 0 ? p.bias_k : p.bias_v) + g * r;

    float acc[kAcc];
#pragma unroll
    for (int u = 0; u < kAcc; ++u) acc[u] = 0.f;

    const int i0 = chunk * kTok;
    for (int k0 = 0; k0 < S; k0 += kK) {
        const int kw = min(kK, S - k0);
        for (int idx = tid; idx < kTok * kK; idx += kThreads) {
            const int ti = idx / kK, kk = idx - ti * kK;
            const int i = i0 + ti;
            float v = 0.f;
            if (i < p.n && kk < kw) {
                size_t off;
                if (p.variant == 0)
                    off = ((((size_t(i) * p.num_layers + L) * p.H + h) * 2 + axis) * S) + k0 + kk;
                else
                    off = (((size_t(i) * p.num_layers + L) * 2 + axis) * S) + k0 + kk;
                v = bf16_to_f32(p.x[off]);
            }
            xs[ti][kk] = v;
        }
        for (int idx = tid; idx < r * kK; idx += kThreads) {
            const int a = idx / kK, kk = idx - a * kK;
            ws[idx] = kk < kw ? bf16_to_f32(W[size_t(a) * S + k0 + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < kK; ++kk) {
            const float xv = xs[tok][kk];
#pragma unroll
            for (int u = 0; u < kAcc; ++u) {
                const int a = agrp + 4 * u;
                if (a < r) acc[u] = fmaf(xv, ws[a * kK + kk], acc[u]);
            }
        }
        __syncthreads();
    }

    const int i = i0 + tok;
    if (i >= p.n) return;
    const int sq = p.seq_idx[i], tk = p.tok_idx[i];
    if (sq < 0 || sq >= p.batch || tk < 0 || tk >= p.max_tokens) return;
    const long long ri = p.smap.row_index(sq, layer, tk, p.D, p.max_tokens);
    if (ri < 0) return;  // a page index out of range: not written
    const size_t row = p.variant == 0 ? size_t(p.H) * (p.r_k + p.r_v) : size_t(p.r_k + p.r_v);
    uint16_t* dst = p.store + size_t(ri) * row +
                    (p.variant == 0 ? size_t(h) * (p.r_k + p.r_v) : 0) + (axis == 0 ? 0 : p.r_k);
#pragma unroll
    for (int u = 0; u < kAcc; ++u) {
        const int a = agrp + 4 * u;
        if (a < r) {
            __nv_bfloat16 v = __float2bfloat16_rn(acc[u] - bias[a]);
            dst[a] = *reinterpret_cast<uint16_t*>(&v);
        }
    }
}

}  // namespace

lla_status lla_encode_launch(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                             const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* store, int batch,
                             int max_tokens, cudaStream_t stream, const lla_store_map& smap) {
    // the tensor-core kernel where it applies (TMA needs 16-byte aligned rows and stacks)
    if ((reinterpret_cast<uintptr_t>(x) & 15) == 0 && (reinterpret_cast<uintptr_t>(store) & 15) == 0) {
        const lla_status st = lla_encode_tc(c, x, n, layer_begin, num_layers, seq_idx, tok_idx, store, batch,
                                            max_tokens, stream, smap);
        if (st != LLA_ERR_UNSUPPORTED_SHAPE) return st;
    }
    return lla_encode_simt(c, x, n, layer_begin, num_layers, seq_idx, tok_idx, store, batch, max_tokens, stream,
                           smap);
}

lla_status lla_encode_simt(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                           const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* store, int batch,
                           int max_tokens, cudaStream_t stream, const lla_store_map& smap) {
    const lla_codec_desc& ds = c->desc;
    if (ds.r_k > kMaxR || ds.r_v > kMaxR) return LLA_ERR_UNSUPPORTED_SHAPE;
    EncodeParams p;
    p.x = x;
    p.seq_idx = seq_idx;
    p.tok_idx = tok_idx;
    p.store = store;
    p.wdt_k = c->w_down_k_t;
    p.wdt_v = c->w_down_v_t;
    p.bias_k = c->bias_k;
    p.bias_v = c->bias_v;
    p.n = n;
    p.layer_begin = layer_begin;
    p.num_layers = num_layers;
    p.H = ds.H;
    p.S = c->S;
    p.r_k = ds.r_k;
    p.r_v = ds.r_v;
    p.variant = ds.variant;
    p.batch = batch;
    p.max_tokens = max_tokens;
    p.D = ds.D;
    p.smap = smap;
    const int rmax = ds.r_k > ds.r_v ? ds.r_k : ds.r_v;
    const size_t smem = size_t(rmax) * kK * sizeof(float);
    LLA_CUDA_TRY(cudaFuncSetAttribute(encode_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    const int Hg = ds.variant == 0 ? ds.H : 1;
    dim3 grid((n + kTok - 1) / kTok, num_layers * Hg, 2);
    encode_simt_kernel<<<grid, kThreads, smem, stream>>>(p);
    LLA_CUDA_TRY(cudaGetLastError());
    return LLA_OK;
}
