// Tensor-core (tcgen05 / TMEM / TMA) LLA decode attention for sm_100a.
//
// What is computed [LLA §3 eq. (3), "RoPE and reconstruction"]: for each
// sequence b and head h at loop t,
//   s_j = scale * < RoPE_{q_pos}(q), RoPE_j(c^K_j W^K_up,t^T + mu^K_t) >,
//   out = sum_j softmax(s)_j (c^V_j W^V_up,t^T + mu^V_t).
//
// How.  With rotate-half RoPE, writing q' = scale * RoPE_{q_pos}(q) and
// Phi_j = [cos(j theta_i) | sin(j theta_i)]_{i < d/2}, the score is bilinear:
//   s_j = Phi_j . (M c^K_j + beta) = sum_a c^K_{j,a} G_{j,a} + G_{j,bias}
// with G = Phi M_q, where the columns of M_q hold, for i < d/2,
//   MA[i,a] = q'_i W[i,a] + q'_{i+d/2} W[i+d/2,a],  MB[i,a] = q'_{i+d/2} W[i,a] - q'_i W[i+d/2,a]
// (and the same with mu in place of W[:,a] for the bias column).  The
// reconstruction and the rotation thus collapse into one [128 x d] x [d x N]
// tcgen05 GEMM per 128-token tile (Phi tile from a codec table, M_q built per
// (sequence, head) by the prologue kernel), and the CUDA cores only do an
// r_k-long dot product per (token, head), the online softmax, and the V side
// in latent space: acc += p_j c^V_j.  The split-combine kernel lifts acc.
//
// Kernel structure (one CTA per SM, persistent over a flattened range of
// (head part, sequence, 128-token tile) work), per-head latents:
//   warp 0      TMA producer of latent stages: per (tile, head, token chunk) a box
//               of (r_k + r_v) x 1 head x TOKS tokens (wide rows: three panels, the
//               c^K ones swizzled) into a ring of shared-memory stages.
//   warp 1      TMEM allocator and MMA issuer: per tile and head group, d/16
//               tcgen05.mma (M=128, N=NG, K=16, fp16 in, fp32 out) into a ring of
//               TMEM buffers, committed to mbarriers.
//   warp 2      (narrow rows) TMA producer of the M_q image per (sequence, head
//               part) and the Phi tile per tile; with wide rows warp 0 does this.
//   the rest    compute: thread = token row (its TMEM lane); the warps of a lane
//               quarter split the heads of each group.  Each keeps (m, l, acc) per
//               head for its 32 rows and writes one record per (segment, quarter,
//               head) for the combine kernel.
// The LLA-2D kernel (decode_tc2d.cuh) shares the walk, the prologue and the records.
// Every wait is bounded (see sm100.cuh); a timeout sets a status bit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "lla_internal.cuh"
#include "sm100.cuh"
#include "walk.cuh"

namespace {

using namespace sm100;
using lla_walk::TileWalker;

constexpr int kTile = 128;
constexpr int kSmemLimit = 232448;  // 227 KB per CTA
constexpr int kMaxCtas = 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kFlagTimeout = 4u;

constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Head grouping shared by both kernels: which heads share one score GEMM (a TMEM group,
// N <= 256 columns), how many groups stay resident per CTA (their M_q images), and so how
// many CTAs ("parts") split the heads of a tile.
template <int DH_, int RK_, int RV_, int H_, int GPC_CAP = 8>
struct HeadGroups {
    static constexpr int DH = DH_, RK = RK_, RV = RV_, H = H_;
    // heads per TMEM group: as many as fit N <= 256 (even, dividing H)
    static constexpr int HG = (16 * (RK + 1) <= 240 && H % 16 == 0) ? 16
                              : (8 * (RK + 1) <= 240 && H % 8 == 0) ? 8
                              : (4 * (RK + 1) <= 240 && H % 4 == 0) ? 4 : 2;
    static constexpr int NG = round_up(HG * RK + HG, 16);
    static constexpr int MQ_GROUP_BYTES = NG * DH * 2;
    static constexpr int GPC_MAX = (110 * 1024) / MQ_GROUP_BYTES;  // resident M_q budget ~110 KB
    static constexpr int GPC_FIT = (H / HG) <= GPC_MAX ? (H / HG) : ((H / HG) % 2 == 0 && GPC_MAX >= 2 ? 2 : 1);
    static constexpr int GPC = GPC_FIT < GPC_CAP ? GPC_FIT : GPC_CAP;
    static constexpr int HC = HG * GPC;  // heads per CTA work item
    static constexpr int PARTS = H / HC;
    static constexpr int MQ_BYTES = GPC * MQ_GROUP_BYTES;
    static constexpr int PHI_BYTES = kTile * DH * 2;
    static constexpr uint32_t IDESC = idesc_f16_f32(128, NG);
    static_assert(DH % 64 == 0 && DH <= 256, "d_head must be a multiple of 64");
    static_assert(H % HC == 0 && HG % 2 == 0, "head split");
};

// Per-head latent rows (one row of r_k + r_v per (token, head)).  Wide rows (512 B and up)
// make a 32-token stage of one head 16 KB: such codecs keep one head group resident (a
// deeper stage ring) and give each lane quarter one compute warp, which walks the heads of
// the item in turn, so that at most four stages are being read while the rest prefetch.
template <int DH_, int RK_, int RV_, int H_, bool WIDE_ = (RK_ + RV_) * 2 >= 512>
struct Cfg : HeadGroups<DH_, RK_, RV_, H_, WIDE_ ? 1 : 8> {
    using HG_ = HeadGroups<DH_, RK_, RV_, H_, WIDE_ ? 1 : 8>;
    using HG_::DH, HG_::RK, HG_::RV, HG_::H, HG_::HG, HG_::NG, HG_::HC, HG_::MQ_BYTES, HG_::PHI_BYTES;
    static constexpr bool TWO_D = false;
    static constexpr bool WIDE = WIDE_;
    static constexpr int ROW = RK + RV;
    static constexpr int TOKS = (ROW * 2 * 128 <= 16384) ? 128 : (ROW * 2 * 64 <= 16384) ? 64 : 32;
    static constexpr int CHUNKS = kTile / TOKS;
    static constexpr int STAGE_BYTES = TOKS * ROW * 2;
    // wide rows land in three panels per stage: c^K elements [0, 64) in the 128-byte swizzle,
    // [64, r_k) in the 64-byte swizzle (bank-conflict-free row reads) and c^V as plain rows
    static constexpr int K0_BYTES = WIDE ? TOKS * 128 : 0;
    static constexpr int K1_BYTES = WIDE ? TOKS * (RK - 64) * 2 : 0;
    static constexpr int V_OFF = K0_BYTES + K1_BYTES;
    static constexpr int BAR_BYTES = 1024;
    static constexpr int FIXED = 1024 /*align slack*/ + PHI_BYTES + MQ_BYTES + BAR_BYTES;
    static constexpr int NST_RAW = (kSmemLimit - FIXED) / STAGE_BYTES;
    static constexpr int NST = NST_RAW > 32 ? 32 : NST_RAW;
    static constexpr int SMEM = FIXED + NST * STAGE_BYTES;
    // compute warps: WPQ per TMEM lane quarter, each taking HG / WPQ heads of every group
    static constexpr int WPQ = WIDE ? 1 : (HG >= 4 ? 4 : HG);
    static constexpr int NCW = 4 * WPQ;
    // warps: latent-stage producer, MMA issuer, (narrow rows) M_q/Phi producer, compute
    static constexpr bool PHI_WARP = !WIDE;
    static constexpr int CW0 = PHI_WARP ? 3 : 2;
    static constexpr int THREADS = 32 * (CW0 + NCW);
    static constexpr int HPW = HC / WPQ;  // heads per compute warp
    // one stage per (head, token chunk), read by that head's warp of each quarter in the chunk
    static constexpr int STAGES_PER_TILE = HC * CHUNKS;
    static constexpr int ST_CONSUMERS = TOKS / 32;
    static constexpr int TMEM_COLS = 512;
    // TMEM accumulator ring: as many NG-column buffers as fit in 512 columns (at most 4)
    static constexpr int NBUF = (512 / NG) > 4 ? 4 : (512 / NG);
    static constexpr int BUF_COLS = (512 / NBUF) / 16 * 16;
    // V-side lane mapping
    static constexpr bool VQUAD = (RV == 32 || RV == 64 || RV == 128);
    static constexpr int VAL = VQUAD ? RV / 4 : 32;          // lanes along the latent dimension
    static constexpr int VTL = 32 / VAL;                      // token sub-lanes
    static constexpr int VPL = VQUAD ? 4 : RV / 16;           // accumulators per lane per head
    // two-token V path (r_v a multiple of 32 outside VQUAD): c^V row pitch in 32-bit words; a
    // pitch that is a multiple of 32 words puts both tokens of a step on the same banks, so
    // the odd token's half-warp takes its words in rotated order
    static constexpr int VPW = WIDE ? RV / 2 : ROW / 2;
    static constexpr bool VROT = VPW % 32 == 0;
    static_assert(RK % 16 == 0 && RV % 32 == 0, "ranks");
    static_assert(HC % WPQ == 0, "head split");
    static_assert(NG <= BUF_COLS, "TMEM buffer");
    static_assert(NST >= 2, "stages");
    static_assert(SMEM <= kSmemLimit, "shared memory");
    static_assert((ROW * 2) % 16 == 0, "TMA row stride");
    static_assert(!WIDE || (RK == 96 && TOKS == 32), "wide rows: c^K split as 64 + 32 elements");
};

// Tensor maps over the layer's latents (the per-head wide layout uses all three).
struct LatMaps {
    CUtensorMap m[3];
};

struct TcParams {
    const uint16_t* phi_tiles;   // codec Phi table, one PHI_BYTES image per 128 positions
    const uint8_t* mq;           // prologue output: M_q images per (part, sequence)
    const int32_t* P;            // tile prefix per sequence [B+1]
    const int32_t* lens;         // clamped lengths [B]
    const float* inv_scale;      // per (b, h): log2(e) / M_q scale
    float* records;              // [(G + PARTS*B)][4][HC][RV+2]
    uint32_t* status;
    int B, G;
    // paged store: tile t of sequence b is pool page table[b * max_pages + t] (null: contiguous)
    const int32_t* table;
    int max_pages, D, layer;
};

static_assert(kTile == kPageTokens, "a tile of a paged store is one page");

// TMA coordinates of tile t of sequence b: the token coordinate of its first row and the outer
// coordinate (sequence, or pool page and layer of a paged store).
__device__ __forceinline__ void tile_coords(const TcParams& p, int b, int t, int& tok0, int& outer) {
    if (p.table) {
        tok0 = 0;
        outer = __ldg(p.table + size_t(b) * p.max_pages + t) * p.D + p.layer;
    } else {
        tok0 = t * kTile;
        outer = b;
    }
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

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) tc_decode_kernel(const __grid_constant__ LatMaps maps,
                                                                TcParams p) {
    const CUtensorMap& lat_map = maps.m[0];
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* phi_s = smem;
    uint8_t* mq_s = phi_s + C::PHI_BYTES;
    uint8_t* stage_s = mq_s + C::MQ_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stage_s + C::NST * C::STAGE_BYTES);
    uint64_t* phi_full = bars;
    uint64_t* phi_empty = bars + 1;
    uint64_t* mq_full = bars + 2;
    uint64_t* mq_empty = mq_full + 1;
    uint64_t* tm_full = mq_full + 2;          // [NBUF]
    uint64_t* tm_empty = tm_full + C::NBUF;  // [NBUF]
    // Round r of stage slot s lands on barrier st_full[r % 4][s].  Compute warps drift apart by
    // up to NBUF head groups (a warp can only start a group once every warp has released the
    // group NBUF before it), which can exceed a ring round: a parity wait on one barrier per
    // slot could then match an earlier round of the slot.  With four barriers per slot a wait
    // could only alias a round four rounds back, which every consumer has long released.
    uint64_t* st_full = tm_empty + C::NBUF;  // [4][NST]
    uint64_t* st_empty = st_full + 4 * C::NST;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(st_empty + C::NST);
    static_assert((4 + 2 * C::NBUF + 5 * C::NST) * 8 + 16 <= C::BAR_BYTES, "barrier area");
    static_assert(C::NBUF * (C::STAGES_PER_TILE / C::GPC) <= 4 * C::NST, "stage rounds a wait can be ahead");
    auto st_full_bar = [&](uint32_t slot, uint32_t round) { return st_full + (round & 3) * C::NST + slot; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(phi_full, 1);
        mbar_init(phi_empty, 1);
        mbar_init(mq_full, 1);
        mbar_init(mq_empty, 1);
        for (int i = 0; i < C::NBUF; ++i) {
            mbar_init(tm_full + i, 1);
            mbar_init(tm_empty + i, C::NCW);
        }
        for (int i = 0; i < 4 * C::NST; ++i) mbar_init(st_full + i, 1);
        for (int i = 0; i < C::NST; ++i) mbar_init(st_empty + i, C::ST_CONSUMERS);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    lla_grid_dependency_wait();  // the prologue's tile plan and M_q images are read from here on

    TileWalker wk;
    wk.init(p.P, p.B, p.G, blockIdx.x, C::PARTS);

    // M_q image on a sequence change and the tile's Phi: issued by the elected thread of the
    // warp that owns them
    uint32_t phi_n = 0, mq_n = 0;
    int mq_key = -1;
    auto phi_mq_step = [&]() -> bool {
        const uint64_t pol_keep = policy_evict_last();
        const int key = wk.key();
        if (key != mq_key) {
            if (mq_n > 0 && !mbar_wait(mq_empty, (mq_n - 1) & 1, p.status, kFlagTimeout, 1)) return false;
            mbar_expect_tx(mq_full, C::MQ_BYTES);
            const uint8_t* src = p.mq + (size_t(wk.p) * p.B + wk.b) * C::MQ_BYTES;
            for (int off = 0; off < C::MQ_BYTES; off += 32768) {
                const int n = C::MQ_BYTES - off < 32768 ? C::MQ_BYTES - off : 32768;
                bulk_g2s(mq_s + off, src + off, n, mq_full, pol_keep);
            }
            ++mq_n;
            mq_key = key;
        }
        if (phi_n > 0 && !mbar_wait(phi_empty, (phi_n - 1) & 1, p.status, kFlagTimeout, 2)) return false;
        mbar_expect_tx(phi_full, C::PHI_BYTES);
        bulk_g2s(phi_s, p.phi_tiles + size_t(wk.t) * (C::PHI_BYTES / 2), C::PHI_BYTES, phi_full, pol_keep);
        ++phi_n;
        return true;
    };
    auto phi_mq_drain = [&]() {
        if (phi_n > 0) mbar_wait(phi_full, (phi_n - 1) & 1, p.status, kFlagTimeout, 5);
        if (mq_n > 0) mbar_wait(mq_full, (mq_n - 1) & 1, p.status, kFlagTimeout, 6);
    };

    // Latent stages of the CTA's walk, in ring order.  With narrow rows the M_q/Phi warp issues
    // the stages of odd heads and warp 0 those of even heads: one issuing thread shares its
    // scheduler with four compute warps, and the loads of a tile went out measurably faster from
    // two (about 4% per call).  With wide rows warp 0 issues every stage and the M_q/Phi loads.
    auto produce = [&](int parity_sel, bool with_phi) {
        prefetch_tensormap(&lat_map);
        if (C::WIDE) {
            prefetch_tensormap(&maps.m[1]);
            prefetch_tensormap(&maps.m[2]);
        }
        const uint64_t pol_stream = policy_evict_first();
        uint32_t stage_k = 0;
        bool ok = true;
        for (; wk.valid() && ok; wk.next()) {
            if (with_phi && !(ok = phi_mq_step())) break;
            int tok0, outer;
            tile_coords(p, wk.b, wk.t, tok0, outer);
            for (int hl = 0; hl < C::HC && ok; ++hl) {
                if (parity_sel >= 0 && (hl & 1) != parity_sel) {
                    stage_k += C::CHUNKS;  // the other producer's head
                    continue;
                }
                const int h = wk.p * C::HC + hl;
                for (int ch = 0; ch < C::CHUNKS; ++ch) {
                    const uint32_t slot = stage_k % C::NST, round = stage_k / C::NST;
                    if (round > 0 && !(ok = mbar_wait(st_empty + slot, (round - 1) & 1, p.status, kFlagTimeout, 3)))
                        break;
                    uint64_t* bar = st_full_bar(slot, round);
                    mbar_expect_tx(bar, C::STAGE_BYTES);
                    uint8_t* dst = stage_s + size_t(slot) * C::STAGE_BYTES;
                    const int tok = tok0 + ch * C::TOKS;
                    if constexpr (C::WIDE) {
                        tma_load_4d(dst, &maps.m[0], 0, h, tok, outer, bar, pol_stream);
                        tma_load_4d(dst + C::K0_BYTES, &maps.m[1], 64, h, tok, outer, bar, pol_stream);
                        tma_load_4d(dst + C::V_OFF, &maps.m[2], C::RK, h, tok, outer, bar, pol_stream);
                    } else {
                        tma_load_4d(dst, &lat_map, 0, h, tok, outer, bar, pol_stream);
                    }
                    ++stage_k;
                }
            }
        }
        // No copy this thread issued may still be in flight when the CTA exits.
        for (uint32_t s = 0; s < C::NST && s < stage_k; ++s) {
            const uint32_t last = stage_k - 1 - ((stage_k - 1 - s) % C::NST);  // last round of slot s
            if (parity_sel >= 0 && ((last % C::STAGES_PER_TILE) / C::CHUNKS & 1) != uint32_t(parity_sel)) continue;
            mbar_wait(st_full_bar(s, last / C::NST), (last / C::NST >> 2) & 1, p.status, kFlagTimeout, 4);
        }
        if (with_phi) phi_mq_drain();
    };

    if (warp == 0) {
        // ------------------------------------------------------------ latent stage producer
        if (elect_one()) produce(C::PHI_WARP ? 0 : -1, !C::PHI_WARP);
    } else if (C::PHI_WARP && warp == 2) {
        // ------------------------------------------------------------ M_q, Phi and odd-head stages
        // (the next tile's Phi goes out as soon as its buffer is free rather than behind the
        // current tile's latent stages)
        if (elect_one()) produce(1, true);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t phi_n = 0, mq_n = 0, gi = 0, mq_commits = 0, phi_commits = 0;
            int prev_key = -1;
            bool ok = true;
            const uint32_t phi_addr = smem_u32(phi_s), mq_addr = smem_u32(mq_s);
            for (; wk.valid() && ok; wk.next()) {
                const int key = wk.key();
                if (key != prev_key) {
                    if (prev_key != -1) {
                        mma_commit(mq_empty);
                        ++mq_commits;
                    }
                    if (!(ok = mbar_wait(mq_full, mq_n & 1, p.status, kFlagTimeout, 7))) break;
                    ++mq_n;
                    prev_key = key;
                }
                if (!(ok = mbar_wait(phi_full, phi_n & 1, p.status, kFlagTimeout, 8))) break;
                ++phi_n;
                tc_fence_after();
                for (int g = 0; g < C::GPC && ok; ++g) {
                    const uint32_t buf = gi % C::NBUF, use = gi / C::NBUF;
                    if (use > 0 && !(ok = mbar_wait(tm_empty + buf, (use - 1) & 1, p.status, kFlagTimeout, 9))) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + buf * C::BUF_COLS;
#pragma unroll
                    for (int kk = 0; kk < C::DH / 16; ++kk) {
                        const uint32_t koff = uint32_t(kk & 3) * 32;  // 16-element K step inside the 64-wide swizzle atom
                        const uint64_t ad = sw128_kmajor_desc(phi_addr + uint32_t(kk >> 2) * (kTile * 128) + koff);
                        const uint64_t bd = sw128_kmajor_desc(mq_addr + g * C::MQ_GROUP_BYTES +
                                                              uint32_t(kk >> 2) * (C::NG * 128) + koff);
                        mma_f16_ss(d_tmem, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(tm_full + buf);
                    ++gi;
                }
                mma_commit(phi_empty);
                ++phi_commits;
            }
            if (prev_key != -1) {
                mma_commit(mq_empty);
                ++mq_commits;
            }
            // The commits' arrivals land in shared memory: see them complete before the CTA exits.
            if (phi_commits > 0) mbar_wait(phi_empty, (phi_commits - 1) & 1, p.status, kFlagTimeout, 10);
            if (mq_commits > 0) mbar_wait(mq_empty, (mq_commits - 1) & 1, p.status, kFlagTimeout, 11);
        }
    } else {
        // ------------------------------------------------------------ compute warps
        const int cw = warp - C::CW0;
        const int qd = warp & 3;        // TMEM lane quarter = token rows [32 qd, 32 qd + 32)
        const int hf = cw >> 2;         // which of the WPQ warps of this quarter
        const int row = 32 * qd + lane;  // tile row of this thread
        const uint32_t lane_addr = uint32_t(32 * qd) << 16;
        const int ch = (32 * qd) / C::TOKS;              // token chunk holding this quarter
        const int srow0 = 32 * qd - ch * C::TOKS;        // first stage row of this warp
        // this warp's heads: hl = hf + WPQ * i (i < HPW) of the CTA item's HC heads; head hl
        // belongs to TMEM group hl / HG.  Heads of a group alternate between the warps of a
        // quarter and each per-head stage is released right after use, so the stages in use
        // stay adjacent in ring order and the rest of the ring keeps prefetching.

        float m[C::HPW], l[C::HPW], acc[C::HPW][C::VPL];
        float isc[C::HPW];  // this warp's heads' score scales for the current sequence
        // the next sequence's length and scales, loaded at the previous sequence change so that
        // their latency is off the first tile (narrow rows only: the wide-row warps carry 16
        // heads and have no registers to spare)
        constexpr bool kPrefetchSeq = !C::WIDE;
        int pf_b = -1, pf_len = 0;
        float pf_isc[kPrefetchSeq ? C::HPW : 1];
        int len = 0;                         // clamped length of the current sequence
        uint32_t gi = 0, tile_n = 0;
        int prev_key = -1;
        long long prev_id = 0;
        bool ok = true;

        // every lane waits on the stage's barrier (no divergent lane-0 branch on the path) and the
        // warp agrees by one vote
        auto wait_stage = [&](uint32_t slot, uint32_t round) {
            ok = __all_sync(0xffffffffu, ok && mbar_wait(st_full_bar(slot, round), (round >> 2) & 1, p.status,
                                                           kFlagTimeout, 13)) && ok;
        };

        auto flush = [&](long long id) {
#pragma unroll
            for (int hw = 0; hw < C::HPW; ++hw) {
                const int hl = hf + C::WPQ * hw;
                float* rec = p.records + ((size_t(id) * 4 + qd) * C::HC + hl) * size_t(C::RV + 2);
                const float lsum = warp_sum(l[hw]);
                float a[C::VPL];
#pragma unroll
                for (int v = 0; v < C::VPL; ++v) {
                    a[v] = acc[hw][v];
                    for (int o = C::VAL; o < 32; o <<= 1) a[v] += __shfl_xor_sync(0xffffffffu, a[v], o);
                }
                if (lane == 0) {
                    rec[0] = (m[hw] == -INFINITY) ? -INFINITY : m[hw] * kLn2;
                    rec[1] = lsum;
                }
                if (C::VQUAD) {
                    if (lane < C::VAL)
#pragma unroll
                        for (int v = 0; v < 4; ++v) rec[2 + 4 * lane + v] = a[v];
                } else {
                    // lane l16 < 16 holds words l16 + 16 k (k < NW) of the even tokens; lane l16 + 16
                    // holds the odd tokens' (in rotated order: its slot k - 1 is word l16 + 16 k)
                    constexpr int NW = C::RV / 32;
#pragma unroll
                    for (int k = 0; k < NW; ++k) {
                        const int ko = C::VROT ? (k == 0 ? NW - 1 : k - 1) : k;
                        const float o0 = __shfl_down_sync(0xffffffffu, acc[hw][2 * ko], 16);
                        const float o1 = __shfl_down_sync(0xffffffffu, acc[hw][2 * ko + 1], 16);
                        if (lane < 16) {
                            rec[2 + 2 * (lane + 16 * k)] = acc[hw][2 * k] + o0;
                            rec[2 + 2 * (lane + 16 * k) + 1] = acc[hw][2 * k + 1] + o1;
                        }
                    }
                }
            }
        };

        for (; wk.valid() && ok; wk.next(), ++tile_n) {
            const int key = wk.key();
            if (key != prev_key) {
                if (prev_key != -1) flush(prev_id);
#pragma unroll
                for (int hw = 0; hw < C::HPW; ++hw) {
                    m[hw] = -INFINITY;
                    l[hw] = 0.f;
#pragma unroll
                    for (int v = 0; v < C::VPL; ++v) acc[hw][v] = 0.f;
                }
                prev_key = key;
                prev_id = wk.record_id();
                if (kPrefetchSeq && pf_b == wk.b) {
#pragma unroll
                    for (int hw = 0; hw < C::HPW; ++hw) isc[hw] = pf_isc[kPrefetchSeq ? hw : 0];
                    len = pf_len;
                } else {
                    const float* isc_row = p.inv_scale + size_t(wk.b) * C::H + wk.p * C::HC;
#pragma unroll
                    for (int hw = 0; hw < C::HPW; ++hw) isc[hw] = __ldg(isc_row + hf + C::WPQ * hw);
                    len = __ldg(p.lens + wk.b);
                }
                if (kPrefetchSeq) {
                    pf_b = wk.b + 1 < p.B ? wk.b + 1 : -1;
                    if (pf_b >= 0) {
                        const float* isc_row = p.inv_scale + size_t(pf_b) * C::H + wk.p * C::HC;
#pragma unroll
                        for (int hw = 0; hw < C::HPW; ++hw) pf_isc[kPrefetchSeq ? hw : 0] = __ldg(isc_row + hf + C::WPQ * hw);
                        pf_len = __ldg(p.lens + pf_b);
                    }
                }
            }
            const int valid = min(kTile, len - wk.t * kTile);
            const bool row_ok = row < valid;
            const int nv = max(0, min(32, valid - 32 * qd));  // valid rows of this warp

#pragma unroll
            for (int g = 0; g < C::GPC; ++g) {
                if (!ok) break;
                const uint32_t buf = gi % C::NBUF, use = gi / C::NBUF;
                ok = __all_sync(0xffffffffu, mbar_wait(tm_full + buf, use & 1, p.status, kFlagTimeout, 12));
                tc_fence_after();
                const uint32_t tcol = tmem_base + lane_addr + buf * C::BUF_COLS;
#pragma unroll
                for (int hw = 0; hw < C::HPW; ++hw) {
                    const int hl = hf + C::WPQ * hw;        // head within the CTA item
                    if (hl / C::HG != g) continue;          // another group's head (warp-uniform)
                    const int hg = hl - g * C::HG;          // head within the group
                    const uint32_t sk = tile_n * C::STAGES_PER_TILE + hl * C::CHUNKS + ch;
                    const uint32_t slot = sk % C::NST;
                    wait_stage(slot, sk / C::NST);
                    const uint8_t* st = stage_s + size_t(slot) * C::STAGE_BYTES;
                    const uint8_t* myrow = st + size_t(srow0 + lane) * (C::ROW * 2);
                    // 16-byte chunk cc of this row's c^K (wide rows: swizzled panels)
                    auto kchunk = [&](int cc) -> uint4 {
                        if constexpr (C::WIDE) {
                            if (cc < 8)
                                return *reinterpret_cast<const uint4*>(st + lane * 128 + ((cc << 4) ^ ((lane & 7) << 4)));
                            return *reinterpret_cast<const uint4*>(st + C::K0_BYTES + lane * 64 +
                                                                   (((cc - 8) << 4) ^ (((lane >> 1) & 3) << 4)));
                        } else {
                            return *reinterpret_cast<const uint4*>(myrow + cc * 16);
                        }
                    };

                    // ---- score: s = c^K . G + bias, G read from TMEM 32 columns at a time;
                    // packed fp32 pairs: two latent dimensions per f32x2 FMA, two chains
                    float bias;
                    tmem_ld<1>(tcol + C::HG * C::RK + hg, &bias);
                    uint64_t s01 = 0, s23 = 0;
#pragma unroll
                    for (int a0 = 0; a0 < C::RK; a0 += 32) {
                        constexpr int W = C::RK < 32 ? C::RK : 32;
                        float gv[W];
#pragma unroll
                        for (int c0 = 0; c0 < W; c0 += 16) tmem_ld<16>(tcol + hg * C::RK + a0 + c0, &gv[c0]);
                        tmem_wait_ld();
#pragma unroll
                        for (int c0 = 0; c0 < W; c0 += 8) {
                            const uint4 u = kchunk((a0 + c0) >> 3);
                            s01 = f2_fma(bf16x2_to_f2(u.x), f2_pack(gv[c0 + 0], gv[c0 + 1]), s01);
                            s23 = f2_fma(bf16x2_to_f2(u.y), f2_pack(gv[c0 + 2], gv[c0 + 3]), s23);
                            s01 = f2_fma(bf16x2_to_f2(u.z), f2_pack(gv[c0 + 4], gv[c0 + 5]), s01);
                            s23 = f2_fma(bf16x2_to_f2(u.w), f2_pack(gv[c0 + 6], gv[c0 + 7]), s23);
                        }
                    }
                    const float2 sp = f2_unpack(s01), sq = f2_unpack(s23);
                    const float s2 = row_ok ? ((sp.x + sp.y) + (sq.x + sq.y) + bias) * isc[hw] : -INFINITY;
                    // ---- online softmax in base 2
                    const float m_new = fmaxf(m[hw], warp_max(s2));
                    const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m[hw] - m_new);
                    const float pj = row_ok ? fast_exp2(s2 - m_new) : 0.f;
                    l[hw] = fmaf(l[hw], alpha, pj);
                    m[hw] = m_new;
#pragma unroll
                    for (int v = 0; v < C::VPL; ++v) acc[hw][v] *= alpha;
                    // ---- V in latent space: acc += p_j c^V_j over this warp's rows
                    if (C::VQUAD) {
                        const int al = lane % C::VAL;
                        const int ts = lane / C::VAL;
                        // interleave token sub-lanes so that the two half-warps read disjoint banks
                        const int tsub = C::VTL == 4 ? ((ts & 1) * 2 + (ts >> 1)) : ts;
                        const uint8_t* vb = st + size_t(srow0 + tsub) * (C::ROW * 2) + (C::RK + 4 * al) * 2;
                        uint64_t v01 = 0, v23 = 0;  // packed fp32 pairs
                        if (nv == 32) {
#pragma unroll
                            for (int j0 = 0; j0 < 32; j0 += C::VTL) {
                                const float pb = __shfl_sync(0xffffffffu, pj, j0 + tsub);
                                const uint2 u = *reinterpret_cast<const uint2*>(vb + j0 * (C::ROW * 2));
                                const uint64_t pp = f2_pack(pb, pb);
                                v01 = f2_fma(pp, bf16x2_to_f2(u.x), v01);
                                v23 = f2_fma(pp, bf16x2_to_f2(u.y), v23);
                            }
                        } else {
                            // rows past the context may hold any bits: their p is 0 but 0 * NaN is
                            // not, so they are skipped rather than weighted
                            for (int j0 = 0; j0 < 32; j0 += C::VTL) {
                                const float pb = __shfl_sync(0xffffffffu, pj, j0 + tsub);
                                if (j0 + tsub < nv) {
                                    const uint2 u = *reinterpret_cast<const uint2*>(vb + j0 * (C::ROW * 2));
                                    const uint64_t pp = f2_pack(pb, pb);
                                    v01 = f2_fma(pp, bf16x2_to_f2(u.x), v01);
                                    v23 = f2_fma(pp, bf16x2_to_f2(u.y), v23);
                                }
                            }
                        }
                        const float2 w01 = f2_unpack(v01), w23 = f2_unpack(v23);
                        acc[hw][0] += w01.x;
                        acc[hw][1] += w01.y;
                        acc[hw][2] += w23.x;
                        acc[hw][3] += w23.y;
                    } else {
                        // two tokens per step: half-warp `hv` takes token j0 + hv, each lane NW
                        // 32-bit words (bf16 pairs) of c^V, word l16 + 16 k (rotated for the odd
                        // token when both rows of a step would meet on the same banks)
                        constexpr int NW = C::RV / 32;
                        const int hv = lane >> 4, l16 = lane & 15;
                        const uint8_t* vbase = C::WIDE ? st + C::V_OFF : st + C::RK * 2;
                        const uint32_t* vw =
                            reinterpret_cast<const uint32_t*>(vbase + size_t(srow0 + hv) * (C::VPW * 4)) + l16;
                        uint64_t va[NW];
#pragma unroll
                        for (int k = 0; k < NW; ++k) va[k] = 0;
                        if (nv == 32) {
#pragma unroll
                            for (int j0 = 0; j0 < 32; j0 += 2) {
                                const float pb = __shfl_sync(0xffffffffu, pj, j0 + hv);
                                const uint64_t pp = f2_pack(pb, pb);
                                const uint32_t* vr = vw + j0 * C::VPW;
#pragma unroll
                                for (int k = 0; k < NW; ++k) {
                                    const int kr = (C::VROT && hv) ? (k + 1 == NW ? 0 : k + 1) : k;
                                    va[k] = f2_fma(pp, bf16x2_to_f2(vr[16 * kr]), va[k]);
                                }
                            }
                        } else {
                            // rows past the context may hold any bits: skipped, not weighted by 0
#pragma unroll
                            for (int j0 = 0; j0 < 32; j0 += 2) {
                                const float pb = __shfl_sync(0xffffffffu, pj, j0 + hv);
                                if (j0 + hv < nv) {
                                    const uint64_t pp = f2_pack(pb, pb);
                                    const uint32_t* vr = vw + j0 * C::VPW;
#pragma unroll
                                    for (int k = 0; k < NW; ++k) {
                                        const int kr = (C::VROT && hv) ? (k + 1 == NW ? 0 : k + 1) : k;
                                        va[k] = f2_fma(pp, bf16x2_to_f2(vr[16 * kr]), va[k]);
                                    }
                                }
                            }
                        }
#pragma unroll
                        for (int k = 0; k < NW; ++k) {
                            const float2 w = f2_unpack(va[k]);
                            acc[hw][2 * k] += w.x;
                            acc[hw][2 * k + 1] += w.y;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(st_empty + slot);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tm_empty + buf);
                ++gi;
            }
        }
        if (prev_key != -1) flush(prev_id);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

#include "decode_tc2d.cuh"

// ---------------------------------------------------------------------------------------------
// Prologue: tile plan and per-(sequence, head) M_q images with their score scales.
// ---------------------------------------------------------------------------------------------

struct ProParams {
    const float* q;
    const int32_t* q_pos;
    const int32_t* seq_lens;
    const float* w_up_k_t;
    const float* rope_cos;
    const float* rope_sin;
    int32_t* P;
    int32_t* lens;
    float* inv_scale;
    uint8_t* mq;
    uint32_t* status;
    int B, D, T, H, DH, RK, RV, HG, NG, HC, GPC, max_tokens, max_pos, layer, loop, variant;
    int pro_wps, pro_spw;  // warps per sequence, sequences per group of warps
    float scale;
    lla_store_map smap;
};

template <class C>
__global__ void __launch_bounds__(256) tc_prologue_kernel(ProParams p) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (blockIdx.x == 0) {
        // exclusive prefix of per-sequence tile counts (clamped lengths)
        __shared__ int32_t carry;
        __shared__ int32_t warp_tot[8];
        if (threadIdx.x == 0) carry = 0;
        __syncthreads();
        for (int base = 0; base < p.B; base += 256) {
            const int b = base + threadIdx.x;
            int n = 0;
            if (b < p.B) {
                n = p.seq_lens[b];
                if (n > p.max_tokens) { n = p.max_tokens; atomicOr(p.status, LLA_FLAG_SEQ_LEN_CLAMPED); }
                if (n > p.max_pos) { n = p.max_pos; atomicOr(p.status, LLA_FLAG_POS_CLAMPED); }
                if (n < 0) n = 0;
                const int nu = p.smap.usable_tokens(b, n);
                if (nu < n) { n = nu; atomicOr(p.status, LLA_FLAG_PAGE_INVALID); }
                p.lens[b] = n;
            }
            const int tiles = (n + kTile - 1) / kTile;
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
            if (b < p.B) p.P[b] = before + v - tiles;
            __syncthreads();
            if (threadIdx.x == 255) carry = before + v;
            __syncthreads();
        }
        if (threadIdx.x == 0) p.P[p.B] = carry;
        return;
    }
    // CTA (head h, run of sequences): W^K_up,t of the head ([n][i], row RK = mu) is copied once
    // into shared memory; the warps then walk the run, pro_wps warps per sequence (its items
    // spread over them) and pro_spw sequences per group of warps.  All the items of a lane share
    // one 8-wide k chunk (d/8 divides 32), so per sequence the lane rotates and scales the 16
    // entries of q it needs (its rotate-half pairs) once and keeps them in registers.
    constexpr int DH = C::DH, RK = C::RK, half = DH / 2, KC = DH / 8;
    constexpr int NITEM = (RK + 1) * KC;  // (row, 8-wide k chunk) items
    static_assert(32 % KC == 0, "a lane's k chunk is the same in every item it takes");
    static_assert(half % 8 == 0, "no k chunk straddles the rotate-half boundary");
    extern __shared__ __align__(16) float pro_smem[];  // W^K_up,t of the head: [RK + 1][DH]
    __shared__ float red[8];
    const int wps = p.pro_wps, sls = 8 / wps, per_cta = sls * p.pro_spw;
    const int k = blockIdx.x - 1;
    const int h = k % C::H, b_first = (k / C::H) * per_cta;
    const int sl = w / wps, wi = w % wps;
    const size_t slot = p.variant == 0 ? (size_t(p.layer) * C::H + h) * p.T + p.loop
                                       : (size_t(p.layer) * p.T + p.loop) * C::H + h;
    {
        const float* wsrc = p.w_up_k_t + slot * size_t(RK + 1) * DH;
        constexpr int NW4 = (RK + 1) * DH / 4;
        for (int e = threadIdx.x; e < NW4; e += 256) lla_cp_async16(pro_smem + 4 * e, wsrc + 4 * e);
    }
    const int k0 = (lane % KC) * 8, i0 = k0 < half ? k0 : k0 - half;  // the lane's k chunk and pairs
    const bool q_vec = (reinterpret_cast<uintptr_t>(p.q) & 15) == 0;   // q rows are d floats apart
    auto ld8 = [](float* v, const float* src, bool vec) {
        if (vec) {
            const float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 4);
            v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
        } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = src[u];
        }
    };
    lla_cp_async_wait_all();
    __syncthreads();
    // A bound on every entry: entry (n, k) is x a + y b (k < d/2) or y a - x b (k >= d/2) with
    // (x, y) = (q'_i, q'_{i+d/2}) and (a, b) = (w_n,i, w_n,i+d/2), so by Cauchy-Schwarz
    // |entry| <= |(x, y)| |(a, b)|.  cw = the largest |(a, b)| over the head's rows.
    float cw2 = 0.f;
    for (int e = threadIdx.x; e < (RK + 1) * half; e += 256) {
        const int n = e / half, i = e - n * half;
        const float wa = pro_smem[n * DH + i], wb = pro_smem[n * DH + i + half];
        cw2 = fmaxf(cw2, wa * wa + wb * wb);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cw2 = fmaxf(cw2, __shfl_xor_sync(0xffffffffu, cw2, o));
    if (lane == 0) red[w] = cw2;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 8; ++j) cw2 = fmaxf(cw2, red[j]);
    const float cw = sqrtf(cw2);
    const int part = h / C::HC, hc = h % C::HC, g = hc / C::HG, hg = hc % C::HG;
    for (int j = 0; j < p.pro_spw; ++j) {
        const int b = b_first + sl + sls * j;
        if (b >= p.B) break;
        int qp = p.q_pos[b];
        if (qp < 0 || qp >= p.max_pos) {
            qp = qp < 0 ? 0 : p.max_pos - 1;
            if (h == 0 && wi == 0 && lane == 0) atomicOr(p.status, LLA_FLAG_POS_CLAMPED);
        }
        // q' = scale * RoPE_qpos(q) on the lane's pairs i0 .. i0 + 8
        const float* qv = p.q + (size_t(b) * C::H + h) * DH;
        float cv[8], sv[8], lo[8], hi[8];
        ld8(cv, p.rope_cos + size_t(qp) * half + i0, true);
        ld8(sv, p.rope_sin + size_t(qp) * half + i0, true);
        ld8(lo, qv + i0, q_vec);
        ld8(hi, qv + i0 + half, q_vec);
        float x[8], y[8];
        float pn = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            x[u] = p.scale * (lo[u] * cv[u] - hi[u] * sv[u]);
            y[u] = p.scale * (hi[u] * cv[u] + lo[u] * sv[u]);
            pn = fmaxf(pn, x[u] * x[u] + y[u] * y[u]);
        }
#pragma unroll
        for (int o = KC / 2; o > 0; o >>= 1) pn = fmaxf(pn, __shfl_xor_sync(0xffffffffu, pn, o));  // every pair
        // power-of-two scale keeping every entry below 2^15 (fp16 then keeps full precision;
        // a power of two changes no rounding, and the scores are divided by it exactly)
        const float bound = sqrtf(pn) * cw;
        float scale = 1.f;
        if (bound > 0.f && isfinite(bound)) {
            int e2 = 0;
            frexpf(bound, &e2);  // bound < 2^e2
            scale = ldexpf(1.f, 15 - max(e2, -100));
        }
        // the lane's entries are pa a + pb b: (pa, pb) = (x, y) for k < d/2, (y, -x) beyond;
        // scaling by a power of two is exact
        const bool upper = k0 >= half;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float xs = x[u] * scale, ys = y[u] * scale;
            x[u] = upper ? ys : xs;
            y[u] = upper ? -xs : ys;
        }
        uint8_t* img = p.mq + (size_t(part) * p.B + b) * size_t(C::MQ_BYTES) + size_t(g) * C::MQ_GROUP_BYTES;
        for (int e = wi * 32 + lane; e < NITEM; e += 32 * wps) {
            const int n = e / KC;  // e % KC == lane % KC
            const float4* wl = reinterpret_cast<const float4*>(pro_smem + n * DH + i0);
            const float4* wh = reinterpret_cast<const float4*>(pro_smem + n * DH + i0 + half);
            const float4 a0 = wl[0], a1 = wl[1], b0 = wh[0], b1 = wh[1];
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
            __align__(16) __half2 hv[4];
#pragma unroll
            for (int u = 0; u < 8; u += 2)
                hv[u / 2] = __floats2half2_rn(x[u] * av[u] + y[u] * bv[u], x[u + 1] * av[u + 1] + y[u + 1] * bv[u + 1]);
            const int rowi = n < RK ? hg * RK + n : C::HG * RK + hg;
            *reinterpret_cast<uint4*>(img + sm100::sw128_offset(rowi, k0, C::NG)) = *reinterpret_cast<const uint4*>(hv);
        }
        if (hg == 0 && wi == 0)  // the group's padding rows
            for (int e = lane; e < (C::NG - C::HG * (RK + 1)) * KC; e += 32) {
                const int rowi = C::HG * (RK + 1) + e / KC, kk = (e % KC) * 8;
                *reinterpret_cast<uint4*>(img + sm100::sw128_offset(rowi, kk, C::NG)) = make_uint4(0, 0, 0, 0);
            }
        if (wi == 0 && lane == 0) p.inv_scale[size_t(b) * C::H + h] = kLog2e / scale;
    }
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
        cudaGetLastError();
    });
    return fn;
}

struct Layout {
    size_t off_P, off_lens, off_isc, off_mq, off_rec, total;
};

template <class C>
Layout tc_layout(int B, int G) {
    Layout L;
    auto al = [](size_t x) { return (x + 1023) & ~size_t(1023); };
    L.off_P = al(sizeof(lla_ws_header));
    L.off_lens = al(L.off_P + size_t(B + 1) * 4);
    L.off_isc = al(L.off_lens + size_t(B) * 4);
    L.off_mq = al(L.off_isc + size_t(B) * C::H * 4);
    L.off_rec = al(L.off_mq + size_t(B) * C::PARTS * C::MQ_BYTES);
    L.total = L.off_rec + (size_t(G) + size_t(C::PARTS) * B) * 4 * C::HC * (C::RV + 2) * sizeof(float);
    return L;
}

template <class C>
int tc_grid(int override_ctas) {
    int g = override_ctas > 0 ? override_ctas : lla_num_sms();
    if (g > kMaxCtas) g = kMaxCtas;
    if (g < C::PARTS) g = C::PARTS;  // at least one CTA per head part
    return g - g % C::PARTS;         // whole groups of parts
}

template <class C>
lla_status run_tc(const lla_decode_call& call, int num_ctas) {
    const lla_codec* c = call.codec;
    const int B = call.batch;
    const int G = tc_grid<C>(num_ctas);
    const Layout L = tc_layout<C>(B, G);
    if (L.total > call.workspace_bytes) return LLA_ERR_WORKSPACE;
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return LLA_ERR_CUDA;
    if ((call.max_tokens + kTile - 1) / kTile > c->phi_num_tiles) return LLA_ERR_UNSUPPORTED_SHAPE;

    char* ws = call.workspace;
    ProParams pp;
    pp.q = call.q;
    pp.q_pos = call.q_pos;
    pp.seq_lens = call.seq_lens;
    pp.w_up_k_t = c->w_up_k_t;
    pp.rope_cos = c->rope_cos;
    pp.rope_sin = c->rope_sin;
    pp.P = reinterpret_cast<int32_t*>(ws + L.off_P);
    pp.lens = reinterpret_cast<int32_t*>(ws + L.off_lens);
    pp.inv_scale = reinterpret_cast<float*>(ws + L.off_isc);
    pp.mq = reinterpret_cast<uint8_t*>(ws + L.off_mq);
    pp.status = reinterpret_cast<uint32_t*>(ws);
    pp.B = B;
    pp.D = c->desc.D;
    pp.T = c->desc.T;
    pp.H = C::H;
    pp.DH = C::DH;
    pp.RK = C::RK;
    pp.RV = C::RV;
    pp.HG = C::HG;
    pp.NG = C::NG;
    pp.HC = C::HC;
    pp.GPC = C::GPC;
    pp.max_tokens = call.max_tokens;
    pp.max_pos = c->desc.max_pos;
    pp.layer = call.layer;
    pp.loop = call.loop;
    pp.variant = c->desc.variant;
    pp.scale = call.scale;
    pp.smap = call.smap;
    // every record the combine reads is written by this call's decode kernel (a CTA writes all
    // of its record set for each sequence it touches; the combine skips groups with no tiles)
    // about four CTAs of eight warps per SM: many sequences run whole on one warp each (and a
    // warp takes several in turn); few are spread over up to eight warps each
    {
        const long long tasks = (long long)B * C::H, target = 32LL * lla_num_sms();
        pp.pro_wps = 1;
        pp.pro_spw = 1;
        if (tasks >= target) pp.pro_spw = int((tasks + target - 1) / target);
        else
            while (pp.pro_wps < 8 && tasks * pp.pro_wps < target) pp.pro_wps *= 2;
    }
    const int pro_per_cta = (8 / pp.pro_wps) * pp.pro_spw;
    const size_t pro_smem = size_t(C::RK + 1) * C::DH * sizeof(float);
    LLA_CUDA_TRY(cudaFuncSetAttribute(tc_prologue_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(pro_smem)));
    tc_prologue_kernel<C><<<1 + C::H * ((B + pro_per_cta - 1) / pro_per_cta), 256, pro_smem, call.stream>>>(pp);
    LLA_CUDA_TRY(cudaGetLastError());

    // Tensor map over the layer's latents: dims (row elems, head, token, sequence).  Per-head
    // rows load whole (r_k + r_v) rows of TOKS tokens; the 2D row loads 64-element panels of
    // 32 tokens in the 128-byte swizzle that the tensor-core operands use.
    // A paged store is addressed as (row elems, head, token of the page, pool page * D + layer).
    const int h_map = C::TWO_D ? 1 : C::H;
    const size_t row_bytes = size_t(h_map) * C::ROW * 2;  // one token of one layer
    LatMaps maps;
    memset(&maps, 0, sizeof(maps));
    const bool paged = call.smap.table != nullptr;
    const void* base = paged ? static_cast<const void*>(call.store)
                             : call.store + size_t(call.layer) * call.max_tokens * (row_bytes / 2);
    cuuint64_t dims[4] = {cuuint64_t(C::ROW), cuuint64_t(h_map),
                          cuuint64_t(paged ? kPageTokens : call.max_tokens),
                          paged ? cuuint64_t(call.smap.num_pages) * c->desc.D : cuuint64_t(B)};
    cuuint64_t strides[3] = {cuuint64_t(C::ROW * 2), cuuint64_t(row_bytes),
                             paged ? cuuint64_t(row_bytes) * kPageTokens
                                   : cuuint64_t(row_bytes) * call.max_tokens * c->desc.D};
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    auto encode = [&](CUtensorMap* m, uint32_t box_elems, uint32_t box_toks, CUtensorMapSwizzle swz) {
        cuuint32_t box[4] = {box_elems, 1u, box_toks, 1u};
        return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    bool enc_ok;
    if constexpr (C::TWO_D) {
        enc_ok = encode(&maps.m[0], 64u, C::QTOK, CU_TENSOR_MAP_SWIZZLE_128B);
    } else if constexpr (C::WIDE) {
        enc_ok = encode(&maps.m[0], 64u, C::TOKS, CU_TENSOR_MAP_SWIZZLE_128B) &&
                 encode(&maps.m[1], C::RK - 64, C::TOKS, CU_TENSOR_MAP_SWIZZLE_64B) &&
                 encode(&maps.m[2], C::RV, C::TOKS, CU_TENSOR_MAP_SWIZZLE_NONE);
    } else {
        enc_ok = encode(&maps.m[0], C::ROW, C::TOKS, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (!enc_ok) return LLA_ERR_CUDA;

    TcParams tp;
    tp.phi_tiles = c->phi_tiles;
    tp.mq = pp.mq;
    tp.P = pp.P;
    tp.lens = pp.lens;
    tp.inv_scale = pp.inv_scale;
    tp.records = reinterpret_cast<float*>(ws + L.off_rec);
    tp.status = pp.status;
    tp.B = B;
    tp.G = G;
    tp.table = call.smap.table;
    tp.max_pages = call.smap.max_pages;
    tp.D = c->desc.D;
    tp.layer = call.layer;
    void (*kernel)(const LatMaps, TcParams);
    if constexpr (C::TWO_D) kernel = tc2d_decode_kernel<C>;
    else kernel = tc_decode_kernel<C>;
    LLA_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    if (call.ev_begin) LLA_CUDA_TRY(cudaEventRecord(call.ev_begin, call.stream));
    // overlapped with the prologue's tail, unless events bracket the kernel for timing
    LLA_CUDA_TRY(lla_launch(kernel, dim3(G), dim3(C::THREADS), C::SMEM, call.stream, call.ev_begin == nullptr, maps, tp));
    if (call.ev_end) LLA_CUDA_TRY(cudaEventRecord(call.ev_end, call.stream));
    lla_tc_ranges ranges;
    ranges.P = pp.P;
    ranges.G = G;
    ranges.parts = C::PARTS;
    ranges.hc = C::HC;
    return lla_combine_tc(call, tp.records, ranges);
}

using CfgRho21 = Cfg<128, 16, 32, 16>;
using CfgRho4 = Cfg<128, 96, 160, 16>;
using Cfg2D = Cfg2<128, 64, 128, 16>;

enum class Which { none, rho21, rho4, two_d };

Which which(const lla_codec* c) {
    const lla_codec_desc& d = c->desc;
    if (d.d_head != 128 || d.H != 16) return Which::none;
    if (d.variant == 1) return (d.r_k == 64 && d.r_v == 128) ? Which::two_d : Which::none;
    if (d.r_k == 16 && d.r_v == 32) return Which::rho21;
    if (d.r_k == 96 && d.r_v == 160) return Which::rho4;
    return Which::none;
}

}  // namespace

bool lla_tc_supported(const lla_codec* c) { return which(c) != Which::none && c->phi_tiles != nullptr; }

size_t lla_tc_workspace_bytes(const lla_codec* c, int batch, int) {
    switch (which(c)) {
        case Which::rho21: return tc_layout<CfgRho21>(batch, kMaxCtas).total;
        case Which::rho4: return tc_layout<CfgRho4>(batch, kMaxCtas).total;
        case Which::two_d: return tc_layout<Cfg2D>(batch, kMaxCtas).total;
        default: return 0;
    }
}

lla_status lla_decode_tc(const lla_decode_call& call, int num_ctas) {
    switch (which(call.codec)) {
        case Which::rho21: return run_tc<CfgRho21>(call, num_ctas);
        case Which::rho4: return run_tc<CfgRho4>(call, num_ctas);
        case Which::two_d: return run_tc<Cfg2D>(call, num_ctas);
        default: return LLA_ERR_UNSUPPORTED_SHAPE;
    }
}

// Phi_j = [cos(j theta_i) | sin(j theta_i)], i < d/2, as fp16 in the tcgen05
// K-major 128-byte-swizzle image, one 128-row tile per 128 positions.
lla_status lla_build_phi_tiles(lla_codec* c, cudaStream_t stream) {
    const int d = c->desc.d_head;
    if (d % 64 != 0 || d > 256) return LLA_OK;  // no tensor-core path for this width
    const int half = d / 2;
    const int tiles = (c->desc.max_pos + kTile - 1) / kTile;
    std::vector<__half> img(size_t(tiles) * kTile * d);
    std::vector<double> theta(half);
    for (int i = 0; i < half; ++i) theta[i] = pow(double(c->desc.rope_base), -2.0 * i / d);
    for (int t = 0; t < tiles; ++t) {
        uint8_t* tile = reinterpret_cast<uint8_t*>(img.data() + size_t(t) * kTile * d);
        for (int r = 0; r < kTile; ++r) {
            const double pos = double(t) * kTile + r;
            for (int k = 0; k < d; ++k) {
                const int i = k < half ? k : k - half;
                const double v = k < half ? cos(pos * theta[i]) : sin(pos * theta[i]);
                *reinterpret_cast<__half*>(tile + sm100::sw128_offset(r, k, kTile)) = __double2half(v);
            }
        }
    }
    if (cudaMalloc(&c->phi_tiles, img.size() * sizeof(__half)) != cudaSuccess) {
        cudaGetLastError();
        c->phi_tiles = nullptr;
        return LLA_ERR_OOM;
    }
    c->phi_num_tiles = tiles;
    if (cudaMemcpyAsync(c->phi_tiles, img.data(), img.size() * sizeof(__half), cudaMemcpyHostToDevice, stream) !=
        cudaSuccess)
        return LLA_ERR_CUDA;
    return cudaStreamSynchronize(stream) == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
}
