// CUDA-core LLA decode attention (no tensor cores): the reference GPU path.
//
// One CTA per (context split, head, sequence).  For each 128-token tile the
// CTA rebuilds loop-t keys k_hat_j = c_j W_up,t^T + mu_t from the cached K
// latents [LLA §3 eq. (3)], rotates them by RoPE at position j and scores
// them against the query rotated to its own position [LLA §3, "RoPE and
// reconstruction"], then keeps an online softmax and sums the V latents
// weighted by p_j in the r_v-dimensional latent space.  The split partials
// (m, l, acc) are merged and up-projected by the combine kernel.
//
// This kernel serves both LLA variants: with the 2D codec the latent row has
// no head axis and W_up / mu are indexed per (loop, head).
#include <math.h>

#include "lla_internal.cuh"

namespace {

constexpr int kThreads = 128;
constexpr int kTile = 128;
static_assert(kTile == kPageTokens, "a tile of a paged store is one page");
constexpr int kMaxRv = 256;  // two accumulators per thread

struct SimtParams {
    const uint16_t* store;
    const float* q;
    const int32_t* q_pos;
    const int32_t* seq_lens;
    const float* w_up_k;
    const float* mu_k;
    const float* rope_cos;
    const float* rope_sin;
    float* partials;
    uint32_t* flags;
    int B, D, H, T, d, r_k, r_v, max_tokens, max_pos, layer, loop, splits, variant;
    float scale;
    lla_store_map smap;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kThreads) simt_decode_kernel(SimtParams p) {
    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = p.d, half = d / 2, rk = p.r_k, rv = p.r_v;

    extern __shared__ float smem[];
    float* W = smem;                 // [d][rk]   W^K_up,t of this head
    float* mu = W + d * rk;          // [d]       mu^K_t
    float* qr = mu + d;              // [d]       scale * RoPE_{q_pos}(q)
    float* cT = qr + d;              // [rk][kTile] K latents, one column per thread
    float* pbuf = cT + rk * kTile;   // [kTile]   softmax numerators of the tile
    float* red = pbuf + kTile;       // [8]       cross-warp reduction scratch

    int n = p.seq_lens[b];
    if (n > p.max_tokens) { n = p.max_tokens; if (tid == 0) atomicOr(p.flags, LLA_FLAG_SEQ_LEN_CLAMPED); }
    if (n > p.max_pos) { n = p.max_pos; if (tid == 0) atomicOr(p.flags, LLA_FLAG_POS_CLAMPED); }
    if (n < 0) n = 0;
    {
        const int nu = p.smap.usable_tokens(b, n);
        if (nu < n) { n = nu; if (tid == 0) atomicOr(p.flags, LLA_FLAG_PAGE_INVALID); }
    }
    int qp = p.q_pos[b];
    if (qp < 0 || qp >= p.max_pos) {
        qp = qp < 0 ? 0 : p.max_pos - 1;
        if (tid == 0) atomicOr(p.flags, LLA_FLAG_POS_CLAMPED);
    }
    const int ntiles = (n + kTile - 1) / kTile;
    const int per = (ntiles + p.splits - 1) / p.splits;
    const int t0 = split * per, t1 = min(ntiles, t0 + per);

    size_t wk_off, mu_off;
    if (p.variant == 0) {
        wk_off = ((size_t(p.layer) * p.H + h) * p.T + p.loop) * size_t(d) * rk;
        mu_off = (size_t(p.layer) * p.H + h) * size_t(p.T) * d + size_t(p.loop) * d;
    } else {
        wk_off = ((size_t(p.layer) * p.T + p.loop) * p.H + h) * size_t(d) * rk;
        mu_off = size_t(p.layer) * p.T * p.H * d + (size_t(p.loop) * p.H + h) * d;
    }
    for (int i = tid; i < d * rk; i += kThreads) W[i] = p.w_up_k[wk_off + i];
    for (int i = tid; i < d; i += kThreads) mu[i] = p.mu_k[mu_off + i];
    const float* qv = p.q + (size_t(b) * p.H + h) * d;
    for (int i = tid; i < half; i += kThreads) {
        const float c = p.rope_cos[size_t(qp) * half + i], s = p.rope_sin[size_t(qp) * half + i];
        const float lo = qv[i], hi = qv[i + half];
        qr[i] = p.scale * (lo * c - hi * s);
        qr[i + half] = p.scale * (hi * c + lo * s);
    }

    const size_t row = p.variant == 0 ? size_t(p.H) * (rk + rv) : size_t(rk + rv);
    const size_t hoff = p.variant == 0 ? size_t(h) * (rk + rv) : 0;

    float m = -INFINITY, l = 0.f, acc0 = 0.f, acc1 = 0.f;
    __syncthreads();

    for (int tile = t0; tile < t1; ++tile) {
        const int j0 = tile * kTile;
        const int cnt = min(kTile, n - j0);
        const int j = j0 + tid;
        // the tile's rows are consecutive (a whole page of a paged store)
        const uint16_t* base = p.store + size_t(p.smap.row_index(b, p.layer, j0, p.D, p.max_tokens)) * row + hoff;
        float s = -INFINITY;
        if (tid < cnt) {
            const uint16_t* cr = base + size_t(tid) * row;
            for (int a = 0; a < rk; ++a) cT[a * kTile + tid] = bf16_to_f32(cr[a]);
            const float* cs = p.rope_cos + size_t(j) * half;
            const float* sn = p.rope_sin + size_t(j) * half;
            float dot = 0.f;
            for (int i = 0; i < half; ++i) {
                float klo = mu[i], khi = mu[i + half];
                const float* wl = W + i * rk;
                const float* wh = W + (i + half) * rk;
                for (int a = 0; a < rk; ++a) {
                    const float ca = cT[a * kTile + tid];
                    klo = fmaf(wl[a], ca, klo);
                    khi = fmaf(wh[a], ca, khi);
                }
                const float c = cs[i], sv = sn[i];
                dot = fmaf(qr[i], klo * c - khi * sv, dot);
                dot = fmaf(qr[i + half], khi * c + klo * sv, dot);
            }
            s = dot;
        }
        // tile maximum across the CTA
        float mx = warp_max(s);
        if (lane == 0) red[warp] = mx;
        __syncthreads();
        mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
        const float m_new = fmaxf(m, mx);
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
        const float pj = (tid < cnt) ? expf(s - m_new) : 0.f;
        pbuf[tid] = pj;
        const float ps = warp_sum(pj);
        __syncthreads();  // red[] reads above are done; pbuf complete
        if (lane == 0) red[4 + warp] = ps;
        __syncthreads();
        l = l * alpha + (red[4] + red[5] + red[6] + red[7]);
        // V side in latent space: acc[a] += sum_j p_j c^V_{j,a}
        {
            const uint16_t* vb = base + rk;
            int a = tid;
            if (a < rv) {
                float v = 0.f;
                for (int jj = 0; jj < cnt; ++jj) v = fmaf(pbuf[jj], bf16_to_f32(vb[size_t(jj) * row + a]), v);
                acc0 = acc0 * alpha + v;
            }
            a += kThreads;
            if (a < rv) {
                float v = 0.f;
                for (int jj = 0; jj < cnt; ++jj) v = fmaf(pbuf[jj], bf16_to_f32(vb[size_t(jj) * row + a]), v);
                acc1 = acc1 * alpha + v;
            }
        }
        m = m_new;
        __syncthreads();  // pbuf / red reused by the next tile
    }

    float* rec = p.partials + ((size_t(b) * p.splits + split) * p.H + h) * lla_partial_floats(rv);
    if (tid == 0) { rec[0] = m; rec[1] = l; }
    if (tid < rv) rec[2 + tid] = acc0;
    if (tid + kThreads < rv) rec[2 + kThreads + tid] = acc1;
}

int simt_splits(int batch, int H, int max_tokens) {
    const int tiles = (max_tokens + kTile - 1) / kTile;
    const int want = 4 * lla_num_sms();
    int s = (want + batch * H - 1) / (batch * H);
    if (s < 1) s = 1;
    if (s > tiles) s = tiles;
    if (s < 1) s = 1;
    return s;
}

}  // namespace

size_t lla_simt_workspace_bytes(const lla_codec* c, int batch, int max_tokens) {
    const int H = c->desc.H;
    // room for the automatic split count, or for up to 8 splits requested explicitly
    const int splits = max(simt_splits(batch, H, max_tokens), min(8, (max_tokens + kTile - 1) / kTile));
    return sizeof(lla_ws_header) + size_t(batch) * splits * H * lla_partial_floats(c->desc.r_v) * sizeof(float);
}

size_t lla_simt_auto_workspace_bytes(const lla_codec* c, int batch, int max_tokens) {
    // exactly what lla_decode_simt(call, 0) checks against: the automatic split count, clamped to
    // the tile count as the launch clamps it
    const int tiles = (max_tokens + kTile - 1) / kTile;
    int splits = simt_splits(batch, c->desc.H, max_tokens);
    if (splits > tiles) splits = tiles > 0 ? tiles : 1;
    return sizeof(lla_ws_header) + size_t(batch) * splits * c->desc.H * lla_partial_floats(c->desc.r_v) * sizeof(float);
}

lla_status lla_decode_simt(const lla_decode_call& call, int splits_override) {
    const lla_codec* c = call.codec;
    const lla_codec_desc& ds = c->desc;
    if (ds.r_v > kMaxRv || ds.r_k > 128 || ds.d_head > 256) return LLA_ERR_UNSUPPORTED_SHAPE;
    const int tiles = (call.max_tokens + kTile - 1) / kTile;
    int splits = splits_override > 0 ? splits_override : simt_splits(call.batch, ds.H, call.max_tokens);
    if (splits > tiles) splits = tiles > 0 ? tiles : 1;
    if (sizeof(lla_ws_header) + size_t(call.batch) * splits * ds.H * lla_partial_floats(ds.r_v) * sizeof(float) >
        call.workspace_bytes)
        return LLA_ERR_WORKSPACE;

    SimtParams p;
    p.store = call.store;
    p.q = call.q;
    p.q_pos = call.q_pos;
    p.seq_lens = call.seq_lens;
    p.w_up_k = c->w_up_k;
    p.mu_k = c->mu_k;
    p.rope_cos = c->rope_cos;
    p.rope_sin = c->rope_sin;
    p.flags = reinterpret_cast<uint32_t*>(call.workspace);
    p.partials = reinterpret_cast<float*>(call.workspace + sizeof(lla_ws_header));
    p.B = call.batch;
    p.D = ds.D;
    p.H = ds.H;
    p.T = ds.T;
    p.d = ds.d_head;
    p.r_k = ds.r_k;
    p.r_v = ds.r_v;
    p.max_tokens = call.max_tokens;
    p.smap = call.smap;
    p.max_pos = ds.max_pos;
    p.layer = call.layer;
    p.loop = call.loop;
    p.splits = splits;
    p.variant = ds.variant;
    p.scale = call.scale;

    const size_t smem = (size_t(ds.d_head) * ds.r_k + 2 * ds.d_head + size_t(ds.r_k) * kTile + kTile + 8) * sizeof(float);
    LLA_CUDA_TRY(cudaFuncSetAttribute(simt_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    dim3 grid(splits, ds.H, call.batch);
    if (call.ev_begin) LLA_CUDA_TRY(cudaEventRecord(call.ev_begin, call.stream));
    simt_decode_kernel<<<grid, kThreads, smem, call.stream>>>(p);
    LLA_CUDA_TRY(cudaGetLastError());
    if (call.ev_end) LLA_CUDA_TRY(cudaEventRecord(call.ev_end, call.stream));
    return lla_combine(call, p.partials, nullptr, splits);
}
