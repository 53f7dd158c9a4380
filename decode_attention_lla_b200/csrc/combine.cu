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
// of W^V_up,t of its slice are copied asynchronously into shared memory, read from global
// memory in their own order (coalesced) and kept row-major at a padded pitch (w_pitch), so
// that the lanes of a warp (one output dimension each) read distinct banks.  Small batches
// split d into 32-row slices to fill the machine, and every CTA of a (head, sequence) then
// merges the records itself (cheap next to the projection); large batches keep all d rows in
// one CTA.
#include <math.h>

#include "lla_internal.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kSeqPerCta = kThreads / 32;  // one warp per sequence
constexpr int kMaxRowsPerLane = 8;         // output dimensions per lane: d <= 256

// Row pitch of the staged W^V_up,t.  r_v a multiple of 4: 4 (mod 32) words, so that eight
// lanes reading 16 bytes each from eight consecutive rows cover the 32 banks once; otherwise
// odd, so that rows i and i + 1 start in different banks.
__host__ __device__ inline int w_pitch(int rv) { return rv % 4 == 0 ? (rv + 27) / 32 * 32 + 4 : rv | 1; }

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
    long long g0, total, groups;
    int b, part, parts, hc;
    // did group g0 + i write its records?  Only a group with an empty tile range writes none,
    // and there is none unless the batch has fewer tiles than there are groups.
    __device__ bool written_group(int i) const {
        if (!tc || total >= groups) return true;
        const int t = int(total), gs = int(groups), g = int(g0) + i;  // total < groups: small
        return t * (g + 1) / gs > t * g / gs;
    }
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
    r.g0 = 0;
    r.total = 0;
    r.groups = 1;
    if (r.tc) {
        r.parts = p.tc_parts;
        r.hc = p.tc_hc;
        r.part = h / p.tc_hc;
        r.hrec = h - r.part * p.tc_hc;
        const long long total = p.tc_P[p.B];
        const int tiles = p.tc_P[b + 1] - p.tc_P[b];
        const long long groups = p.tc_G / p.tc_parts;
        if (tiles == 0 || total == 0 || groups == 0) return r;
        r.total = total;
        r.groups = groups;
        const long long x0 = p.tc_P[b], x1 = x0 + tiles - 1;
        long long g1;
        if ((x1 + 1) * groups < (1LL << 32)) {  // the usual sizes: 32-bit divisions
            r.g0 = uint32_t((x0 + 1) * groups - 1) / uint32_t(total);
            g1 = uint32_t((x1 + 1) * groups - 1) / uint32_t(total);
        } else {
            r.g0 = ((x0 + 1) * groups - 1) / total;
            g1 = ((x1 + 1) * groups - 1) / total;
        }
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

// One warp per (sequence, head); the CTA's eight warps share the rows of W^V_up,t of one head.
// A lane holds NC latent dimensions (a = lane + 32 c, c < NC, 32 NC >= r_v) and RPL output
// rows (32 RPL >= the CTA's rows).  The warp's loads go out in as few dependent rounds as the
// data allows: W (asynchronous copies into shared memory) before the wait for the decode
// kernel, then the record set's bounds, then every record's (m, l) together with the acc of the
// first kRC records; the merge and the projection then run from registers and shared memory.
template <int NC, int RPL>
__global__ void __launch_bounds__(kThreads, 3) combine_kernel(CombineParams p) {
    constexpr int kRC = NC <= 2 ? 8 : 16 / NC >= 2 ? 16 / NC : 2;  // records whose acc a lane holds at once
    const int h = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y * kSeqPerCta + warp;
    const bool active = b < p.B;
    const int d = p.d, rv = p.r_v, pitch = w_pitch(rv);
    const int rows = d / gridDim.z;  // output dimensions of this CTA's slice (gridDim.z divides d)
    const int i0 = blockIdx.z * rows;
    extern __shared__ __align__(16) float smem[];
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
    {
        // W is read in its own (coalesced) order; each element (four of them when r_v is a multiple
        // of 4: rows and pitch then keep 16-byte alignment) lands at its padded place
        const float* wg = p.w_up_v + w_off + size_t(i0) * rv;
        const int vec = rv % 4 == 0 ? 4 : 1, rw = rv / vec, nw = rows * rw;
        int r = threadIdx.x / rw, a = threadIdx.x - (threadIdx.x / rw) * rw;
        const int dr = kThreads / rw, da = kThreads - (kThreads / rw) * rw;
        for (int e = threadIdx.x; e < nw; e += kThreads) {
            if (vec == 4) lla_cp_async16(Ws + r * pitch + 4 * a, wg + 4 * e);
            else lla_cp_async4(Ws + r * pitch + a, wg + e);
            r += dr;
            a += da;
            if (a >= rw) {
                a -= rw;
                ++r;
            }
        }
    }
    lla_grid_dependency_wait();  // W is a constant; the records come from the decode kernel

    const size_t bh = size_t(b) * p.H + h;
    float L = 0.f, w_self = 0.f;
    if (active) {
        const RecordSet rs = record_set(p, b, h);
        const int n = rs.n;
        // groups of the record set that wrote records (a group whose tile range is empty did
        // not): one bit per group for the first 32 groups, computed directly beyond
        uint32_t wmask = 0xffffffffu;
        if (rs.tc) wmask = __ballot_sync(0xffffffffu, lane * 4 < n && rs.written_group(lane));
        auto written = [&](int s) { return s / 4 < 32 ? ((wmask >> (s / 4)) & 1u) != 0 : rs.written_group(s / 4); };
        // records go in blocks of 32, record sb + j of a block on lane j: its address, (m, l) and
        // weight are that lane's, and reach the warp by shuffle
        auto shfl_ptr = [&](const float* q, int j) -> const float* {
            const uint64_t u = reinterpret_cast<uint64_t>(q);
            const uint32_t lo = __shfl_sync(0xffffffffu, uint32_t(u), j), hi = __shfl_sync(0xffffffffu, uint32_t(u >> 32), j);
            return reinterpret_cast<const float*>((uint64_t(hi) << 32) | lo);
        };
        const float* my = rs.rec(lane < n ? lane : 0);
        // one round: (m, l) of record `lane` and the acc of records [0, kRC)
        float m0 = -INFINITY, l0 = 0.f;
        if (lane < n && written(lane)) {
            m0 = my[0];
            l0 = my[1];
        }
        float x0[kRC][NC];
#pragma unroll
        for (int j = 0; j < kRC; ++j) {
            const bool use = j < n && written(j);
            const float* r = shfl_ptr(my, j) + 2 + lane;
#pragma unroll
            for (int c = 0; c < NC; ++c) x0[j][c] = (use && lane + 32 * c < rv) ? r[32 * c] : 0.f;
        }
        // self-slot logit (natural-log units, like the records' m)
        float s_self = -INFINITY;
        if (p.k_self) {
            float dot = 0.f;
            for (int i = lane; i < d; i += 32) dot = fmaf(p.q[bh * d + i], p.k_self[bh * d + i], dot);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            s_self = p.scale * dot;
        }
        // log-sum-exp over the records: a lane-wise running merge, then across the warp; a
        // record with l = 0 saw no valid token and is skipped whatever its m holds
        float mx = -INFINITY, sx = 0.f;
        auto merge = [&](float ms, float ls) {
            if (!(ls > 0.f)) return;
            if (ms > mx) {
                sx = sx * expf(mx - ms) + ls;
                mx = ms;
            } else {
                sx += ls * expf(ms - mx);
            }
        };
        merge(m0, l0);
#pragma unroll 1
        for (int s = lane + 32; s < n; s += 32)
            if (written(s)) {
                const float* r = rs.rec(s);
                merge(r[0], r[1]);
            }
        float M = mx;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        M = fmaxf(M, s_self);
        L = sx > 0.f ? sx * expf(mx - M) : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        const float e_self = p.k_self ? expf(s_self - M) : 0.f;
        L += e_self;
        const float invL = L > 0.f ? 1.f / L : 0.f;
        w_self = e_self * invL;
        // abar = sum_s w_s acc_s with w_s = exp(m_s - M) / L
        const float w0 = l0 > 0.f ? expf(m0 - M) * invL : 0.f;
        float v[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) v[c] = 0.f;
#pragma unroll
        for (int j = 0; j < kRC; ++j) {
            const float wj = __shfl_sync(0xffffffffu, w0, j);
#pragma unroll
            for (int c = 0; c < NC; ++c) v[c] = fmaf(x0[j][c], wj, v[c]);
        }
#pragma unroll 1
        for (int sb = 0; sb < n; sb += 32) {
            const float* mine = my;
            float wb = w0;
            if (sb > 0) {
                const int s = sb + lane;
                mine = rs.rec(s < n ? s : sb);
                wb = 0.f;
                if (s < n && written(s) && mine[1] > 0.f) wb = expf(mine[0] - M) * invL;
            }
            const int nb = min(32, n - sb);
#pragma unroll 1
            for (int j0 = sb == 0 ? kRC : 0; j0 < nb; j0 += kRC) {
                float x[kRC][NC];
#pragma unroll
                for (int j = 0; j < kRC; ++j) {
                    const int jj = (j0 + j) & 31;
                    const bool use = j0 + j < nb && written(sb + jj);
                    const float* r = shfl_ptr(mine, jj) + 2 + lane;
#pragma unroll
                    for (int c = 0; c < NC; ++c) x[j][c] = (use && lane + 32 * c < rv) ? r[32 * c] : 0.f;
                }
#pragma unroll
                for (int j = 0; j < kRC; ++j) {
                    const float wj = __shfl_sync(0xffffffffu, wb, (j0 + j) & 31);
#pragma unroll
                    for (int c = 0; c < NC; ++c) v[c] = fmaf(x[j][c], wj, v[c]);
                }
            }
        }
#pragma unroll
        for (int c = 0; c < NC; ++c)
            if (lane + 32 * c < rv) abar[lane + 32 * c] = v[c];
    }
    lla_cp_async_wait_all();
    __syncthreads();  // W staged by every thread of the CTA
    if (!active) return;
    float* o = p.out + bh * d;
    if (!(L > 0.f)) {  // empty context
        for (int r = lane; r < rows; r += 32) o[i0 + r] = 0.f;
        return;
    }
    // out_i = abar . W^V_up,t[i] + (1 - w_self) mu^V_t[i] + w_self v_self[i] for i = i0 + r,
    // r = lane + 32 k; the rows of a lane keep independent accumulation chains
    float acc[RPL], muv[RPL];  // mu of the lane's rows: loaded under the projection's arithmetic
#pragma unroll
    for (int k = 0; k < RPL; ++k) {
        acc[k] = 0.f;
        muv[k] = lane + 32 * k < rows ? __ldg(p.mu_v + mu_off + i0 + lane + 32 * k) : 0.f;
    }
    const float* wr = Ws + size_t(min(lane, rows - 1)) * pitch;
    const int nk = (rows + 31) / 32;
    if (RPL <= 4 && rv == 32 * NC && rows == 32 * RPL) {  // whole blocks: no guards, fixed offsets
#pragma unroll 4
        for (int a = 0; a < 32 * NC; a += 4) {
            const float4 x = *reinterpret_cast<const float4*>(abar + a);
#pragma unroll
            for (int k = 0; k < RPL; ++k) {
                const float4 w = *reinterpret_cast<const float4*>(wr + 32 * k * pitch + a);
                acc[k] = fmaf(x.x, w.x, acc[k]);
                acc[k] = fmaf(x.y, w.y, acc[k]);
                acc[k] = fmaf(x.z, w.z, acc[k]);
                acc[k] = fmaf(x.w, w.w, acc[k]);
            }
        }
    } else if (rv % 4 == 0) {  // 16-byte reads of W rows and of abar (pitch and rv multiples of 4)
#pragma unroll 2
        for (int a = 0; a < rv; a += 4) {
            const float4 x = *reinterpret_cast<const float4*>(abar + a);
#pragma unroll
            for (int k = 0; k < RPL; ++k)
                if (k < nk && lane + 32 * k < rows) {
                    const float4 w = *reinterpret_cast<const float4*>(wr + size_t(32 * k) * pitch + a);
                    acc[k] = fmaf(x.x, w.x, acc[k]);
                    acc[k] = fmaf(x.y, w.y, acc[k]);
                    acc[k] = fmaf(x.z, w.z, acc[k]);
                    acc[k] = fmaf(x.w, w.w, acc[k]);
                }
        }
    } else {
        for (int a = 0; a < rv; ++a) {
            const float x = abar[a];
#pragma unroll
            for (int k = 0; k < RPL; ++k)
                if (k < nk && lane + 32 * k < rows) acc[k] = fmaf(x, wr[size_t(32 * k) * pitch + a], acc[k]);
        }
    }
#pragma unroll
    for (int k = 0; k < RPL; ++k) {
        const int r = lane + 32 * k;
        if (k >= nk || r >= rows) break;
        const int i = i0 + r;
        o[i] = acc[k] + (p.k_self ? fmaf(w_self, p.v_self[bh * d + i], (1.f - w_self) * muv[k]) : muv[k]);
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
    if (ds.d_head > 32 * kMaxRowsPerLane || ds.r_v > 256) return LLA_ERR_UNSUPPORTED_SHAPE;
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
    void (*kernel)(CombineParams) = nullptr;
    const int rows = ds.d_head / z;  // rows per lane: 2, 4 or 8 blocks of 32
    switch ((ds.r_v + 31) / 32) {
#define LLA_COMBINE_CASE(nc)                                                                        \
    case nc:                                                                                        \
        kernel = rows <= 64 ? combine_kernel<nc, 2> : rows <= 128 ? combine_kernel<nc, 4> : combine_kernel<nc, 8>; \
        break;
        LLA_COMBINE_CASE(1)
        LLA_COMBINE_CASE(2)
        LLA_COMBINE_CASE(3)
        LLA_COMBINE_CASE(4)
        LLA_COMBINE_CASE(5)
        LLA_COMBINE_CASE(6)
        LLA_COMBINE_CASE(7)
        LLA_COMBINE_CASE(8)
#undef LLA_COMBINE_CASE
        default: return LLA_ERR_UNSUPPORTED_SHAPE;
    }
    LLA_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    dim3 grid(ds.H, seq_ctas, z);
    // overlapped with the decode kernel's tail, unless an event follows that kernel for timing
    LLA_CUDA_TRY(lla_launch(kernel, grid, dim3(kThreads), smem, call.stream, call.ev_end == nullptr, p));
    return LLA_OK;
}
