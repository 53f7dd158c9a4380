// Comparator: decode attention over a full (uncompressed) bf16 K/V cache.
//
// The latent store is contrasted with a "fast path" that keeps every cached token's loop-t key
// and value themselves [LLA summary, "Serving Capacity"; LLA §3, "Teacher cache"].  This is
// that path's decode for one (layer, loop) call, built for the same machine, so that the two
// can be timed side by side where the full cache fits:
//   s_j = scale * <RoPE_{q_pos}(q), k_j>   (keys cached already rotated at their positions)
//   out = sum_j softmax(s)_j v_j,          zero for an empty context.
// Per (token, head) it reads 4 d bytes and does 2 d FMAs: an HBM-bound GEMV, so the dot
// products stay on the CUDA cores and the design is about keeping enough bytes in flight.
//
// Layout: k_cache, v_cache bf16 [batch][H][max_tokens][d] (head-major: each (sequence, head)
// stream is contiguous, so the walk below streams whole DRAM rows) with a sequence stride
// (elements) that may exceed H * max_tokens * d (a slice of a larger [batch][layers][loops][...]
// cache).
//
// Kernels:
//   full_prologue   block 0: clamped lengths and the tile prefix over the B*H (sequence,
//                   head) streams; the other blocks: q' = scale * RoPE(q) in fp32 from
//                   double-precision angles.
//   full_decode     persistent CTAs over the flattened (stream, 128-token tile) space.  Warp 0
//                   issues TMA per (tile, 32-token quarter): K as two 64-element panels in
//                   the 128-byte swizzle (each thread then reads its own key row without bank
//                   conflicts), V as plain rows, into a ring of 12 stages of 16 KB.  Compute
//                   warp q takes quarter q of every tile, so it waits only on its own stages
//                   while the rest of the ring keeps loading: the score with thread = token
//                   and q' broadcast from shared memory, the value sum with lane = 4
//                   dimensions, each over four independent accumulation chains (one warp per
//                   SM sub-partition has no other warp to hide a dependent FMA's latency).
//                   Each warp keeps (m, l, acc[d]) per stream segment and writes one record.
//   full_combine    one warp per (sequence, head): log-sum-exp merge, out = acc / L.
// Every wait is bounded; a timeout sets a status bit.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include "lla_internal.cuh"
#include "sm100.cuh"
#include "walk.cuh"

namespace {

using namespace sm100;
using lla_walk::TileWalker;

constexpr int kTile = 128;
constexpr int kD = 128;                  // head width this kernel is built for
constexpr int kQ = 32;                   // tokens per stage: a quarter of a tile
constexpr int kQuarters = kTile / kQ;
constexpr int kSets = 1;                 // compute warp sets, taking alternate tiles (two sets measured slower)
constexpr int kCW = kSets * kQuarters;   // compute warps
constexpr int kThreads = 32 * (1 + kCW);
constexpr int kMaxRegs = 240;            // two warps' registers fit one SM sub-partition
constexpr int kPanel = kQ * 128;         // one 64-element swizzled K panel of a quarter
constexpr int kKBytes = 2 * kPanel;      // K of a quarter
constexpr int kVBytes = kQ * kD * 2;     // V of a quarter
constexpr int kStage = kKBytes + kVBytes;
constexpr int kNST = 12;
constexpr int kSmem = 1024 + kNST * kStage + 1024 + kCW * kD * 4;
constexpr int kRec = kCW;                // records per (CTA, stream) segment: one per compute warp
constexpr int kRecF = kD + 4;            // record floats: m, l, 2 pad, acc[kD] (acc 16-byte aligned)
constexpr int kMaxCtas = 1024;
constexpr uint32_t kFlagTimeout = 4u;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
static_assert(kSmem <= 232448, "shared memory");

struct FullParams {
    const float* q;
    const int32_t* q_pos;
    const int32_t* seq_lens;
    int32_t* P;     // [B*H + 1] tile prefix over streams s = b*H + h
    int32_t* lens;  // [B]
    float* qr;      // [B][H][d] scale * RoPE(q), log2(e) folded in
    float* records; // [(G + B*H)][kRec][kRecF]
    uint32_t* status;
    int B, H, max_tokens, G;
    float scale;
    double rope_base;
};

__global__ void __launch_bounds__(256) full_prologue(FullParams p) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (blockIdx.x == 0) {
        __shared__ int32_t carry;
        __shared__ int32_t warp_tot[8];
        if (threadIdx.x == 0) carry = 0;
        for (int b = threadIdx.x; b < p.B; b += 256) {
            int n = p.seq_lens[b];
            if (n > p.max_tokens) { n = p.max_tokens; atomicOr(p.status, LLA_FLAG_SEQ_LEN_CLAMPED); }
            if (n < 0) n = 0;
            p.lens[b] = n;
        }
        __syncthreads();
        const int S = p.B * p.H;
        for (int base = 0; base < S; base += 256) {
            const int s = base + threadIdx.x;
            const int tiles = s < S ? (p.lens[s / p.H] + kTile - 1) / kTile : 0;
            int v = tiles;  // inclusive warp scan
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += y;
            }
            if (lane == 31) warp_tot[w] = v;
            __syncthreads();
            int before = carry;
            for (int i = 0; i < w; ++i) before += warp_tot[i];
            if (s < S) p.P[s] = before + v - tiles;
            __syncthreads();
            if (threadIdx.x == 255) carry = before + v;
            __syncthreads();
        }
        if (threadIdx.x == 0) p.P[S] = carry;
        return;
    }
    // q' = scale * log2(e) * RoPE_{q_pos}(q): one thread per rotate-half pair
    const long long idx = (long long)(blockIdx.x - 1) * 256 + threadIdx.x;
    const int half = kD / 2;
    if (idx >= (long long)p.B * p.H * half) return;
    const int i = int(idx % half);
    const long long bh = idx / half;
    const int b = int(bh / p.H);
    int qp = p.q_pos[b];
    if (qp < 0) qp = 0;
    const double ang = double(qp) * pow(p.rope_base, -2.0 * i / kD);
    double sn, cs;
    sincos(ang, &sn, &cs);
    const float* qv = p.q + bh * kD;
    const float lo = qv[i], hi = qv[i + half];
    const float c = float(cs), s = float(sn), f = p.scale * kLog2e;
    p.qr[bh * kD + i] = f * (lo * c - hi * s);
    p.qr[bh * kD + i + half] = f * (hi * c + lo * s);
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float warp_max(float v) { return warp_max_f32(v); }
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __maxnreg__(kMaxRegs) full_decode(const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap vmap, FullParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float* qbuf = reinterpret_cast<float*>(ring + kNST * kStage);  // [kCW][kD] each warp's q'
    uint64_t* full = reinterpret_cast<uint64_t*>(qbuf + kCW * kD);
    uint64_t* empty = full + kNST;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNST; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);  // the warp of the quarter
        }
        fence_mbar_init();
    }
    __syncthreads();
    lla_grid_dependency_wait();  // the prologue's tile plan and q' are read from here on

    TileWalker wk;
    wk.init(p.P, p.B * p.H, p.G, blockIdx.x, 1);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (elect_one()) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
            const uint64_t pol = policy_evict_first();
            uint32_t n = 0;  // stages issued
            bool ok = true;
            for (; wk.valid() && ok; wk.next()) {
                const int b = wk.b / p.H, h = wk.b - b * p.H;
                for (int q = 0; q < kQuarters; ++q, ++n) {
                    const uint32_t slot = n % kNST, round = n / kNST;
                    if (round > 0 && !(ok = mbar_wait(empty + slot, (round - 1) & 1, p.status, kFlagTimeout, 1)))
                        break;
                    mbar_expect_tx(full + slot, kStage);
                    uint8_t* st = ring + size_t(slot) * kStage;
                    const int tok = wk.t * kTile + q * kQ;
                    tma_load_4d(st, &kmap, 0, tok, h, b, full + slot, pol);
                    tma_load_4d(st + kPanel, &kmap, 64, tok, h, b, full + slot, pol);
                    tma_load_4d(st + kKBytes, &vmap, 0, tok, h, b, full + slot, pol);
                }
            }
            for (uint32_t s = 0; s < kNST && s < n; ++s) {  // nothing in flight at exit
                const uint32_t last = n - 1 - ((n - 1 - s) % kNST);
                mbar_wait(full + s, (last / kNST) & 1, p.status, kFlagTimeout, 2);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- compute warps
    const int cw = warp - 1;
    const int set = cw / kQuarters;  // tiles n of the walk with n % kSets == set
    const int qd = cw % kQuarters;   // token rows [32 qd, 32 qd + 32) of those tiles
    float* qw = qbuf + cw * kD;  // this warp's copy of q', reloaded per stream
    float m = -INFINITY, l = 0.f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};  // dimensions 4 lane .. 4 lane + 3
    uint32_t n = 0;
    int prev = -1;
    bool ok = true;

    auto flush = [&](int s) {
        const int rec_id = int(blockIdx.x) + s;
        float* r = p.records + (size_t(rec_id) * kRec + cw) * kRecF;
        const float lsum = warp_sum(l);
        if (lane == 0) {
            r[0] = (m == -INFINITY) ? -INFINITY : m * kLn2;
            r[1] = lsum;
        }
        *reinterpret_cast<float4*>(r + 4 + 4 * lane) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    };

    for (; wk.valid() && ok; wk.next(), ++n) {
        const int s = wk.b;
        if (s != prev) {
            if (prev != -1) flush(prev);
            m = -INFINITY;
            l = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = 0.f;
            __syncwarp();
            reinterpret_cast<float4*>(qw)[lane] = __ldg(reinterpret_cast<const float4*>(p.qr + size_t(s) * kD) + lane);
            __syncwarp();
            prev = s;
        }
        if (int(n % kSets) != set) continue;  // the other set's tile
        const uint32_t sn = n * kQuarters + qd;  // this warp's stage of the tile
        const uint32_t slot = sn % kNST, round = sn / kNST;
        // The slot cannot be refilled before this warp releases it, so the phase parity alone
        // identifies the fill of this round.
        ok = __all_sync(0xffffffffu, mbar_wait(full + slot, round & 1, p.status, kFlagTimeout, 4)) && ok;
        if (!ok) break;
        const uint8_t* st = ring + size_t(slot) * kStage;
        const int valid = min(kTile, __ldg(p.lens + s / p.H) - wk.t * kTile);
        const int nv = max(0, min(32, valid - 32 * qd));

        // ---- score of this thread's token: 16 swizzled 16-byte chunks of its key row
        uint64_t sa[4] = {0, 0, 0, 0};  // four independent accumulation chains
        const uint8_t* krow = st + lane * 128;
        const uint32_t xr = uint32_t(lane & 7) << 4;
#pragma unroll
        for (int c = 0; c < kD / 8; ++c) {
            const uint4 u = *reinterpret_cast<const uint4*>(krow + (c >> 3) * kPanel + ((uint32_t(c & 7) << 4) ^ xr));
            const float4 qa = reinterpret_cast<const float4*>(qw)[2 * c];      // same address in every lane
            const float4 qb = reinterpret_cast<const float4*>(qw)[2 * c + 1];
            sa[0] = f2_fma(bf16x2_to_f2(u.x), f2_pack(qa.x, qa.y), sa[0]);
            sa[1] = f2_fma(bf16x2_to_f2(u.y), f2_pack(qa.z, qa.w), sa[1]);
            sa[2] = f2_fma(bf16x2_to_f2(u.z), f2_pack(qb.x, qb.y), sa[2]);
            sa[3] = f2_fma(bf16x2_to_f2(u.w), f2_pack(qb.z, qb.w), sa[3]);
        }
        const float2 a0 = f2_unpack(sa[0]), a1 = f2_unpack(sa[1]), a2 = f2_unpack(sa[2]), a3 = f2_unpack(sa[3]);
        const bool row_ok = lane < nv;
        const float sc = row_ok ? ((a0.x + a0.y) + (a1.x + a1.y)) + ((a2.x + a2.y) + (a3.x + a3.y)) : -INFINITY;
        const float m_new = fmaxf(m, warp_max(sc));
        const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m - m_new);
        const float pj = row_ok ? fast_exp2(sc - m_new) : 0.f;
        l = fmaf(l, alpha, pj);
        m = m_new;
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] *= alpha;

        // ---- value sum over this warp's 32 rows: lane = dimensions 4 lane .. 4 lane + 3
        const uint8_t* vb = st + kKBytes + 8 * lane;
        uint64_t va[4] = {0, 0, 0, 0};  // dimension pairs (0,1), (2,3) of even and odd rows
        if (nv == 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float pb = __shfl_sync(0xffffffffu, pj, j);
                const uint2 u = *reinterpret_cast<const uint2*>(vb + j * (kD * 2));
                const uint64_t pp = f2_pack(pb, pb);
                va[2 * (j & 1)] = f2_fma(pp, bf16x2_to_f2(u.x), va[2 * (j & 1)]);
                va[2 * (j & 1) + 1] = f2_fma(pp, bf16x2_to_f2(u.y), va[2 * (j & 1) + 1]);
            }
        } else {
            // rows past the context may hold any bits: skipped, not weighted by 0
            for (int j = 0; j < nv; ++j) {
                const float pb = __shfl_sync(0xffffffffu, pj, j);
                const uint2 u = *reinterpret_cast<const uint2*>(vb + j * (kD * 2));
                const uint64_t pp = f2_pack(pb, pb);
                va[0] = f2_fma(pp, bf16x2_to_f2(u.x), va[0]);
                va[1] = f2_fma(pp, bf16x2_to_f2(u.y), va[1]);
            }
        }
        const float2 w0 = f2_unpack(va[0]), w1 = f2_unpack(va[1]), w2 = f2_unpack(va[2]), w3 = f2_unpack(va[3]);
        acc[0] += w0.x + w2.x;
        acc[1] += w0.y + w2.y;
        acc[2] += w1.x + w3.x;
        acc[3] += w1.y + w3.y;
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + slot);
    }
    if (prev != -1) flush(prev);
}

// One warp per (sequence, head): merge the records of the CTAs that covered the stream.
__global__ void __launch_bounds__(256) full_combine(FullParams p, float* out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    lla_grid_dependency_wait();  // the records come from the decode kernel
    const long long s = (long long)blockIdx.x * 8 + warp;
    if (s >= (long long)p.B * p.H) return;
    float4* o = reinterpret_cast<float4*>(out + s * kD) + lane;
    const long long total = p.P[p.B * p.H];
    const int x0 = p.P[s], tiles = p.P[s + 1] - x0;
    if (tiles == 0 || total == 0) {
        *o = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }
    // the CTA that owns tile x of the walk: ((x + 1) G - 1) / total
    const long long c0 = ((x0 + 1) * (long long)p.G - 1) / total;
    const long long c1 = ((x0 + tiles) * (long long)p.G - 1) / total;
    const int nrec = int(c1 - c0 + 1) * kRec;
    auto rec = [&](int i) { return p.records + (size_t(c0 + i / kRec + s) * kRec + i % kRec) * kRecF; };
    float M = -INFINITY;
    for (int i = lane; i < nrec; i += 32) {
        const float* r = rec(i);
        if (r[1] > 0.f) M = fmaxf(M, r[0]);
    }
    M = warp_max(M);
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
    if (M != -INFINITY)
        for (int i = 0; i < nrec; ++i) {
            const float* r = rec(i);
            if (!(r[1] > 0.f)) continue;
            const float w = expf(r[0] - M);
            L = fmaf(r[1], w, L);
            const float4 v = *reinterpret_cast<const float4*>(r + 4 + 4 * lane);
            a.x = fmaf(v.x, w, a.x);
            a.y = fmaf(v.y, w, a.y);
            a.z = fmaf(v.z, w, a.z);
            a.w = fmaf(v.w, w, a.w);
        }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    *o = make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
}

struct FullLayout {
    size_t off_P, off_lens, off_qr, off_rec, total;
};

FullLayout full_layout(int B, int H, int G) {
    auto al = [](size_t x) { return (x + 1023) & ~size_t(1023); };
    FullLayout L;
    L.off_P = al(sizeof(lla_ws_header));
    L.off_lens = al(L.off_P + (size_t(B) * H + 1) * 4);
    L.off_qr = al(L.off_lens + size_t(B) * 4);
    L.off_rec = al(L.off_qr + size_t(B) * H * kD * 4);
    L.total = L.off_rec + (size_t(G) + size_t(B) * H) * kRec * kRecF * sizeof(float);
    return L;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn full_encode_fn() {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(f);
}

}  // namespace

size_t lla_full_workspace_bytes(int H, int batch) { return full_layout(batch, H, kMaxCtas).total; }

lla_status lla_full_decode(int H, float rope_base, const uint16_t* k_cache, const uint16_t* v_cache,
                           long long seq_stride, int batch, int max_tokens, const float* q, const int32_t* q_pos,
                           const int32_t* seq_lens, float scale, float* out, void* workspace, size_t workspace_bytes,
                           int num_ctas, cudaStream_t stream) {
    int G = num_ctas > 0 ? num_ctas : lla_num_sms();
    if (G > kMaxCtas) G = kMaxCtas;
    const FullLayout L = full_layout(batch, H, G);
    if (L.total > workspace_bytes) return LLA_ERR_WORKSPACE;
    EncodeTiledFn enc = full_encode_fn();
    if (!enc) return LLA_ERR_CUDA;
    char* ws = static_cast<char*>(workspace);
    FullParams p;
    p.q = q;
    p.q_pos = q_pos;
    p.seq_lens = seq_lens;
    p.P = reinterpret_cast<int32_t*>(ws + L.off_P);
    p.lens = reinterpret_cast<int32_t*>(ws + L.off_lens);
    p.qr = reinterpret_cast<float*>(ws + L.off_qr);
    p.records = reinterpret_cast<float*>(ws + L.off_rec);
    p.status = reinterpret_cast<uint32_t*>(ws);
    p.B = batch;
    p.H = H;
    p.max_tokens = max_tokens;
    p.G = G;
    p.scale = scale;
    p.rope_base = rope_base;
    LLA_CUDA_TRY(cudaMemsetAsync(workspace, 0, sizeof(lla_ws_header), stream));
    LLA_CUDA_TRY(cudaMemsetAsync(p.records, 0, L.total - L.off_rec, stream));
    const long long pairs = (long long)batch * H * (kD / 2);
    full_prologue<<<1 + int((pairs + 255) / 256), 256, 0, stream>>>(p);
    LLA_CUDA_TRY(cudaGetLastError());

    // (d, token, head, sequence); K in two 64-element panels with the 128-byte swizzle
    cuuint64_t dims[4] = {cuuint64_t(kD), cuuint64_t(max_tokens), cuuint64_t(H), cuuint64_t(batch)};
    cuuint64_t strides[3] = {cuuint64_t(kD) * 2, cuuint64_t(max_tokens) * kD * 2, cuuint64_t(seq_stride) * 2};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    cuuint32_t kbox[4] = {64u, uint32_t(kQ), 1u, 1u}, vbox[4] = {uint32_t(kD), uint32_t(kQ), 1u, 1u};
    CUtensorMap kmap, vmap;
    if (enc(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(k_cache), dims, strides, kbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        enc(&vmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t*>(v_cache), dims, strides, vbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return LLA_ERR_CUDA;
    LLA_CUDA_TRY(cudaFuncSetAttribute(full_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
    // each kernel is scheduled while its predecessor drains and waits for its results
    LLA_CUDA_TRY(lla_launch(full_decode, dim3(G), dim3(kThreads), kSmem, stream, true, kmap, vmap, p));
    LLA_CUDA_TRY(lla_launch(full_combine, dim3(int((batch * (long long)H + 7) / 8)), dim3(256), 0, stream, true, p, out));
    return LLA_OK;
}
