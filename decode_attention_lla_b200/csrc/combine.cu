// Split-combine and V up-projection for LLA decode attention.
//
// Every split of a sequence's context leaves a record (m, l, acc[r_v]) per
// head: its running maximum score, the sum of exp(s_j - m), and
// sum_j exp(s_j - m) c^V_j in the r_v-dimensional latent space.  The records
// are merged by log-sum-exp and the merged latent a = acc / l is lifted once:
//   out = a W^V_up,t^T + mu^V_t,
// which equals sum_j p_j v_hat_j because the normalised p_j sum to one
// [LLA §3 eq. (3)].  An empty context (no records with l > 0) yields zeros.
//
// One CTA per (head, 16 sequences), one warp per sequence: W^V_up,t of the head
// is staged in shared memory once, transposed so that the lanes of a warp (one
// output dimension each) read consecutive words.
#include <math.h>

#include "lla_internal.cuh"

namespace {

constexpr int kThreads = 512;
constexpr int kSeqPerCta = kThreads / 32;  // one warp per sequence

struct CombineParams {
    const float* partials;
    const int32_t* slot_range;  // [B][2] (begin, end) or null: slots b*splits .. +splits
    const float* w_up_v;
    const float* mu_v;
    float* out;
    int B, H, T, d, r_v, layer, loop, splits, variant;
    // tensor-core record layout (tc_P != null): see lla_tc_ranges
    const int32_t* tc_P;
    int tc_G, tc_parts, tc_hc;
};

// Record range [s0, s1) and record stride for (b, h).  In the tensor-core
// layout, CTA c of G covers flattened tiles [c W / G, (c+1) W / G) with
// W = parts * total; the CTA owning tile x is ((x + 1) G - 1) / W.
__device__ __forceinline__ void record_range(const CombineParams& p, int b, int h, int& s0, int& s1, int& hrec,
                                             int& hstride) {
    if (p.tc_P) {
        const int part = h / p.tc_hc;
        hrec = h - part * p.tc_hc;
        hstride = p.tc_hc;
        const long long total = p.tc_P[p.B];
        const int tiles = p.tc_P[b + 1] - p.tc_P[b];
        if (tiles == 0 || total == 0) {
            s0 = s1 = 0;
            return;
        }
        const long long W = total * p.tc_parts;
        const long long x0 = part * total + p.tc_P[b], x1 = x0 + tiles - 1;
        const long long c0 = ((x0 + 1) * p.tc_G - 1) / W, c1 = ((x1 + 1) * p.tc_G - 1) / W;
        const long long key = (long long)part * p.B + b;
        s0 = int(4 * (key + c0));
        s1 = int(4 * (key + c1 + 1));
    } else if (p.slot_range) {
        s0 = p.slot_range[2 * b];
        s1 = p.slot_range[2 * b + 1];
        hrec = h;
        hstride = p.H;
    } else {
        s0 = b * p.splits;
        s1 = s0 + p.splits;
        hrec = h;
        hstride = p.H;
    }
}

// One warp per (sequence, head); the CTA's sixteen warps share W^V_up,t of one head.
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineParams p) {
    const int h = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y * kSeqPerCta + warp;
    const int d = p.d, rv = p.r_v;
    extern __shared__ float smem[];
    float* Wt = smem;                     // [rv][d]
    float* mu = Wt + rv * d;              // [d]
    float* abar = mu + d + warp * rv;     // [kSeqPerCta][rv]

    size_t w_off, mu_off;
    if (p.variant == 0) {
        w_off = ((size_t(p.layer) * p.H + h) * p.T + p.loop) * size_t(d) * rv;
        mu_off = (size_t(p.layer) * p.H + h) * size_t(p.T) * d + size_t(p.loop) * d;
    } else {
        w_off = ((size_t(p.layer) * p.T + p.loop) * p.H + h) * size_t(d) * rv;
        mu_off = size_t(p.layer) * p.T * p.H * d + (size_t(p.loop) * p.H + h) * d;
    }
    // transposed into shared memory: consecutive threads write consecutive i (no bank conflicts)
    for (int idx = threadIdx.x; idx < d * rv; idx += blockDim.x) {
        const int a = idx / d, i = idx - a * d;
        Wt[idx] = __ldg(p.w_up_v + w_off + size_t(i) * rv + a);
    }
    for (int i = threadIdx.x; i < d; i += blockDim.x) mu[i] = __ldg(p.mu_v + mu_off + i);
    __syncthreads();
    if (b >= p.B) return;

    const size_t rec_len = lla_partial_floats(rv);
    int s0, s1, hr, hs;
    record_range(p, b, h, s0, s1, hr, hs);
    auto rec = [&](int s) { return p.partials + (size_t(s) * hs + hr) * rec_len; };
    // merged maximum and normaliser over the records (log-sum-exp); a record with l = 0
    // saw no valid token and is skipped whatever its m holds
    float M = -INFINITY;
    for (int s = s0 + lane; s < s1; s += 32) {
        const float* r = rec(s);
        if (r[1] > 0.f) M = fmaxf(M, r[0]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    if (M != -INFINITY)
        for (int s = s0 + lane; s < s1; s += 32) {
            const float* r = rec(s);
            if (r[1] > 0.f) L += r[1] * expf(r[0] - M);
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    float* o = p.out + (size_t(b) * p.H + h) * d;
    if (!(L > 0.f)) {  // empty context
        for (int i = lane; i < d; i += 32) o[i] = 0.f;
        return;
    }
    // record weights exp(m_s - M) / L, one per lane, broadcast by shuffle
    const float invL = 1.f / L;
    for (int a = lane; a < rv; a += 32) abar[a] = 0.f;
    for (int sb = s0; sb < s1; sb += 32) {
        float wgt = 0.f;
        if (sb + lane < s1) {
            const float* r = rec(sb + lane);
            if (r[1] > 0.f) wgt = expf(r[0] - M) * invL;
        }
        const int ns = min(32, s1 - sb);
        for (int a0 = 0; a0 < rv; a0 += 32) {  // whole warp in every iteration (shuffles)
            const int a = a0 + lane;
            float v = a < rv ? abar[a] : 0.f;
#pragma unroll 4
            for (int j = 0; j < ns; ++j) {
                const float wj = __shfl_sync(0xffffffffu, wgt, j);
                if (wj != 0.f && a < rv) v = fmaf(rec(sb + j)[2 + a], wj, v);
            }
            if (a < rv) abar[a] = v;
        }
    }
    __syncwarp();
    // out = abar W^V_up,t^T + mu^V_t
    for (int i = lane; i < d; i += 32) {
        float v = mu[i];
        for (int a = 0; a < rv; ++a) v = fmaf(abar[a], Wt[a * d + i], v);
        o[i] = v;
    }
}

}  // namespace

static lla_status launch_combine(const lla_decode_call& call, CombineParams& p);

lla_status lla_combine(const lla_decode_call& call, const float* partials, const int32_t* slot_range,
                       int splits) {
    CombineParams p;
    p.partials = partials;
    p.slot_range = slot_range;
    p.splits = splits;
    p.tc_P = nullptr;
    p.tc_G = p.tc_parts = p.tc_hc = 0;
    return launch_combine(call, p);
}

lla_status lla_combine_tc(const lla_decode_call& call, const float* records, const lla_tc_ranges& r) {
    CombineParams p;
    p.partials = records;
    p.slot_range = nullptr;
    p.splits = 0;
    p.tc_P = r.P;
    p.tc_G = r.G;
    p.tc_parts = r.parts;
    p.tc_hc = r.hc;
    return launch_combine(call, p);
}

static lla_status launch_combine(const lla_decode_call& call, CombineParams& p) {
    const lla_codec_desc& ds = call.codec->desc;
    p.w_up_v = call.codec->w_up_v;
    p.mu_v = call.codec->mu_v;
    p.out = call.out;
    p.B = call.batch;
    p.H = ds.H;
    p.T = ds.T;
    p.d = ds.d_head;
    p.r_v = ds.r_v;
    p.layer = call.layer;
    p.loop = call.loop;
    p.variant = ds.variant;
    const size_t smem = (size_t(ds.r_v) * ds.d_head + ds.d_head + size_t(kSeqPerCta) * ds.r_v) * sizeof(float);
    LLA_CUDA_TRY(cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    dim3 grid(ds.H, (call.batch + kSeqPerCta - 1) / kSeqPerCta);
    combine_kernel<<<grid, kThreads, smem, call.stream>>>(p);
    LLA_CUDA_TRY(cudaGetLastError());
    return LLA_OK;
}
