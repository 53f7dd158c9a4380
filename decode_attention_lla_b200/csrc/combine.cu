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
// Optional self slot: the current token's exact loop-t key and value join the softmax as one
// more term.  Query and self key sit at the same position, so their rotations cancel and the
// logit is scale * <q, k_self>; with w_self its normalised weight,
//   out = (sum_s w_s acc_s) W^V_up,t^T + (1 - w_self) mu^V_t + w_self v_self,
// since the cached tokens then carry 1 - w_self of the probability.
//
// One CTA per (head, 8 sequences, slice of output dimensions), one warp per sequence: the rows
// of W^V_up,t of its slice are staged in shared memory, read from global memory in their own
// order (coalesced) and kept row-major with an odd row pitch, so that the lanes of a warp (one
// output dimension each at a time) read distinct banks.  Small batches split d into 32-row
// slices to fill the machine, and every CTA of a (head, sequence) then merges the records
// itself (cheap next to the projection); large batches keep all d rows in one CTA.
#include <math.h>

#include "lla_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kSeqPerCta = kThreads / 32;  // one warp per sequence
constexpr int kMaxRowsPerLane = 8;         // output dimensions per lane and pass
constexpr int kAC = 8;                     // latent dims per lane held in registers while merging

// Row pitch of the staged W^V_up,t: odd, so rows i and i + 1 start in different banks.
__host__ __device__ inline int w_pitch(int rv) { return rv | 1; }

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
    // self slot (k_self == null: none)
    const float* q;
    const float* k_self;
    const float* v_self;
    float scale;
};

// The records of (b, h): rec(s) for s in [0, n).
//   Split kernel: slots b*splits .. (b+1)*splits (or slot_range), record (slot * H + h).
//   Tensor-core kernel: the CTAs form G/parts groups over the tile space; group g covers
//   tiles [g total / groups, (g+1) total / groups), so the group owning tile x is
//   ((x + 1) groups - 1) / total.  Group g's CTA for head part p writes record set
//   id = (g + b) * parts + p, one record per TMEM lane quarter and head of the part:
//   record ((id * 4 + quarter) * hc + head_in_part).
struct RecordSet {
    const float* base;
    size_t rec_len;
    int n;
    // split kernel
    int s0, hstride, hrec;
    // tensor-core kernel
    bool tc;
    long long g0;
    int b, part, parts, hc;
    __device__ const float* rec(int s) const {
        if (!tc) return base + (size_t(s0 + s) * hstride + hrec) * rec_len;
        const long long id = (g0 + s / 4 + b) * parts + part;
        return base + (size_t(id * 4 + (s & 3)) * hc + hrec) * rec_len;
    }
};

__device__ __forceinline__ RecordSet record_set(const CombineParams& p, int b, int h) {
    RecordSet r;
    r.base = p.partials;
    r.rec_len = lla_partial_floats(p.r_v);
    r.tc = p.tc_P != nullptr;
    r.b = b;
    r.n = 0;
    if (r.tc) {
        r.parts = p.tc_parts;
        r.hc = p.tc_hc;
        r.part = h / p.tc_hc;
        r.hrec = h - r.part * p.tc_hc;
        const long long total = p.tc_P[p.B];
        const int tiles = p.tc_P[b + 1] - p.tc_P[b];
        const long long groups = p.tc_G / p.tc_parts;
        if (tiles == 0 || total == 0 || groups == 0) return r;
        const long long x0 = p.tc_P[b], x1 = x0 + tiles - 1;
        r.g0 = ((x0 + 1) * groups - 1) / total;
        const long long g1 = ((x1 + 1) * groups - 1) / total;
        r.n = int(4 * (g1 - r.g0 + 1));
    } else {
        r.hstride = p.H;
        r.hrec = h;
        if (p.slot_range) {
            r.s0 = p.slot_range[2 * b];
            r.n = p.slot_range[2 * b + 1] - r.s0;
        } else {
            r.s0 = b * p.splits;
            r.n = p.splits;
        }
    }
    return r;
}

// One warp per (sequence, head); the CTA's eight warps share 32 rows of W^V_up,t of one head.
__global__ void __launch_bounds__(kThreads, 4) combine_kernel(CombineParams p) {
    const int h = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y * kSeqPerCta + warp;
    const int d = p.d, rv = p.r_v, pitch = w_pitch(rv);
    const int rows = d / gridDim.z;  // output dimensions of this CTA's slice (gridDim.z divides d)
    const int i0 = blockIdx.z * rows;
    extern __shared__ float smem[];
    float* Ws = smem;                         // [rows][pitch]: row r holds W^V_up,t[i0 + r][0..rv)
    float* abar = Ws + rows * pitch + warp * rv;  // [kSeqPerCta][rv]

    size_t w_off, mu_off;
    if (p.variant == 0) {
        w_off = ((size_t(p.layer) * p.H + h) * p.T + p.loop) * size_t(d) * rv;
        mu_off = (size_t(p.layer) * p.H + h) * size_t(p.T) * d + size_t(p.loop) * d;
    } else {
        w_off = ((size_t(p.layer) * p.T + p.loop) * p.H + h) * size_t(d) * rv;
        mu_off = size_t(p.layer) * p.T * p.H * d + (size_t(p.loop) * p.H + h) * d;
    }
    const float* wg = p.w_up_v + w_off + size_t(i0) * rv;
    const int nw = rows * rv;
    if ((rv & 3) == 0 && (reinterpret_cast<uintptr_t>(wg) & 15) == 0) {
        // four consecutive elements of one row per load (rv % 4 == 0: no load spans two rows)
#pragma unroll 4
        for (int e = 4 * threadIdx.x; e < nw; e += 4 * kThreads) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(wg + e));
            const int r = e / rv, a = e - r * rv;
            float* w = Ws + size_t(r) * pitch + a;
            w[0] = v.x;
            w[1] = v.y;
            w[2] = v.z;
            w[3] = v.w;
        }
    } else {
#pragma unroll 4
        for (int e = threadIdx.x; e < nw; e += kThreads) {
            const int r = e / rv, a = e - r * rv;
            Ws[size_t(r) * pitch + a] = __ldg(wg + e);
        }
    }
    __syncthreads();
    lla_grid_dependency_wait();  // W above is a constant; the records come from the decode kernel
    if (b >= p.B) return;

    const RecordSet rs = record_set(p, b, h);
    auto rec = [&](int s) { return rs.rec(s); };
    const int s0 = 0, s1 = rs.n;
    const size_t bh = size_t(b) * p.H + h;
    // self-slot logit (natural-log units, like the records' m)
    float s_self = -INFINITY;
    if (p.k_self) {
        float dot = 0.f;
        for (int i = lane; i < d; i += 32) dot = fmaf(p.q[bh * d + i], p.k_self[bh * d + i], dot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        s_self = p.scale * dot;
    }
    // merged maximum and normaliser over the records (log-sum-exp); a record with l = 0
    // saw no valid token and is skipped whatever its m holds
    float M = s_self;
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
    const float e_self = p.k_self ? expf(s_self - M) : 0.f;
    L += e_self;
    float* o = p.out + bh * d;
    if (!(L > 0.f)) {  // empty context
        for (int r = lane; r < rows; r += 32) o[i0 + r] = 0.f;
        return;
    }
    const float w_self = e_self / L;
    // abar = sum_s w_s acc_s with w_s = exp(m_s - M) / L; record weights one per lane, broadcast
    // by shuffle; lane owns latent dims a0 + lane + 32 c, kAC of them per pass over the records
    const float invL = 1.f / L;
    for (int a0 = 0; a0 < rv; a0 += 32 * kAC) {
        float v[kAC];
#pragma unroll
        for (int c = 0; c < kAC; ++c) v[c] = 0.f;
        for (int sb = s0; sb < s1; sb += 32) {
            float wgt = 0.f;
            if (sb + lane < s1) {
                const float* r = rec(sb + lane);
                if (r[1] > 0.f) wgt = expf(r[0] - M) * invL;
            }
            const int ns = min(32, s1 - sb);
#pragma unroll 2
            for (int j = 0; j < ns; ++j) {
                const float wj = __shfl_sync(0xffffffffu, wgt, j);
                if (wj == 0.f) continue;  // an empty record: its acc is not read
                const float* r = rec(sb + j) + 2 + a0 + lane;
#pragma unroll
                for (int c = 0; c < kAC; ++c)
                    if (a0 + lane + 32 * c < rv) v[c] = fmaf(r[32 * c], wj, v[c]);
            }
        }
#pragma unroll
        for (int c = 0; c < kAC; ++c)
            if (a0 + lane + 32 * c < rv) abar[a0 + lane + 32 * c] = v[c];
    }
    __syncwarp();
    // out_i = abar . W^V_up,t[i] + (1 - w_self) mu^V_t[i] + w_self v_self[i] for i = i0 + r,
    // r = r0 + lane + 32 k; the rows of a lane keep independent accumulation chains
    for (int r0 = 0; r0 < rows; r0 += 32 * kMaxRowsPerLane) {
        float acc[kMaxRowsPerLane];
#pragma unroll
        for (int k = 0; k < kMaxRowsPerLane; ++k) acc[k] = 0.f;
        const float* wr = Ws + size_t(min(r0 + lane, rows - 1)) * pitch;
        const int nk = min(kMaxRowsPerLane, (rows - r0 + 31) / 32);
        for (int a = 0; a < rv; ++a) {
            const float x = abar[a];
#pragma unroll
            for (int k = 0; k < kMaxRowsPerLane; ++k)
                if (k < nk && r0 + lane + 32 * k < rows) acc[k] = fmaf(x, wr[size_t(32 * k) * pitch + a], acc[k]);
        }
#pragma unroll
        for (int k = 0; k < kMaxRowsPerLane; ++k) {
            const int r = r0 + lane + 32 * k;
            if (k >= nk || r >= rows) break;
            const int i = i0 + r;
            const float m = __ldg(p.mu_v + mu_off + i);
            o[i] = acc[k] + (p.k_self ? fmaf(w_self, p.v_self[bh * d + i], (1.f - w_self) * m) : m);
        }
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
    p.q = call.q;
    p.k_self = call.k_self;
    p.v_self = call.v_self;
    p.scale = call.scale;
    // split d into 32-row slices while the grid is short of two CTAs per SM
    const int seq_ctas = (call.batch + kSeqPerCta - 1) / kSeqPerCta;
    int z = 1;
    while (ds.d_head % (64 * z) == 0 && ds.H * seq_ctas * z < 2 * lla_num_sms()) z *= 2;
    const size_t smem = (size_t(w_pitch(ds.r_v)) * (ds.d_head / z) + size_t(kSeqPerCta) * ds.r_v) * sizeof(float);
    LLA_CUDA_TRY(cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    dim3 grid(ds.H, seq_ctas, z);
    // overlapped with the decode kernel's tail, unless an event follows that kernel for timing
    LLA_CUDA_TRY(lla_launch(combine_kernel, grid, dim3(kThreads), smem, call.stream, call.ev_end == nullptr, p));
    return LLA_OK;
}
