// Tensor-core LLA encode: c = (x - mu) W_down = x W_down - b  [LLA §3 eq. (2)].
//
// Persistent CTAs over the work items (128-token tile, layer, head), slot-major so that the CTAs
// running at the same time share W_down's tiles in L2.  For an item, the loop stacks x of the
// tile (K axis and V axis, S = T*d_head each, or T*H*d_head for LLA-2D) are the A operand and
// W_down^T of the two axes the B operands of tcgen05.mma (bf16 in, fp32 accumulators in TMEM:
// r_k columns for K, r_v for V).  K is walked in 64-element chunks staged by TMA with the
// 128-byte swizzle into a ring of shared-memory stages that runs on across items.  Two TMEM
// accumulator buffers let the MMAs of the next item run while four epilogue warps (thread =
// token row) subtract b = mu W_down, round to bf16 (nearest-even) and write each token's
// K || V latent row to the store slot (seq_idx[i], tok_idx[i]).
//
//   warp 0  TMA producer        warp 1  TMEM allocator + MMA issuer
//   warps 2-5  epilogue
// Waits are bounded (sm100.cuh); a wait that gives up sets a bit in the
// codec's status word and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "lla_internal.cuh"
#include "sm100.cuh"

namespace {

using namespace sm100;

constexpr int kTok = 128;
constexpr int kKc = 64;  // K elements per stage (one 128-byte swizzle atom)
constexpr int kThreads = 192;
constexpr int kSmemLimit = 232448;

constexpr int pow2_at_least(int x) {
    int p = 32;
    while (p < x) p <<= 1;
    return p;
}

template <int RK_, int RV_>
struct ECfg {
    static constexpr int RK = RK_, RV = RV_;
    static constexpr int TOK = kTok;  // tokens per work item
    static constexpr int A_BYTES = kTok * kKc * 2;  // one axis' stacks of the 128 tokens, 64 K elements
    static constexpr int BK_BYTES = RK * kKc * 2;
    static constexpr int BV_BYTES = RV * kKc * 2;
    static constexpr int STAGE = 2 * A_BYTES + BK_BYTES + BV_BYTES;  // [A_K | A_V | W_K | W_V]
    // two CTAs per SM when two stages fit in half the shared memory, else one CTA with up to 4 stages
    static constexpr int NST2 = (kSmemLimit / 2 - 2048) / STAGE;
    static constexpr int NST1 = (kSmemLimit - 2048) / STAGE;
    static constexpr int NST = NST2 >= 2 ? (NST2 > 4 ? 4 : NST2) : (NST1 > 4 ? 4 : NST1);
    static constexpr int CTAS_PER_SM = NST2 >= 2 ? 2 : 1;
    static constexpr bool WIDE = false;
    static constexpr int SMEM = 1024 + NST * STAGE + 1024;
    static constexpr int VCOL = (RK + 31) / 32 * 32;  // TMEM column of the V accumulator
    static constexpr int ACC_COLS = pow2_at_least(VCOL + RV);  // one accumulator buffer
    static constexpr int TMEM_COLS = 2 * ACC_COLS;              // two: epilogue and MMA overlap
    static constexpr uint32_t IDESC_K = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(RK >> 3) << 17) | (uint32_t(128 >> 4) << 24);
    static constexpr uint32_t IDESC_V = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(RV >> 3) << 17) | (uint32_t(128 >> 4) << 24);
    static_assert(RK % 16 == 0 && RV % 16 == 0 && RK <= 256 && RV <= 256, "ranks");
    static_assert(TMEM_COLS * CTAS_PER_SM <= 512, "TMEM");
    static_assert(SMEM <= kSmemLimit, "shared memory");
};

struct EncParams {
    const int32_t* seq_idx;
    const int32_t* tok_idx;
    uint16_t* store;
    const float* bias_k;  // [D][Hg][r_k]
    const float* bias_v;
    uint32_t* status;
    int n, layer_begin, num_layers, Hg, S, D, batch, max_tokens, ntiles, nitems;
    size_t row;  // elements per (sequence, layer, token) row of the store
    lla_store_map smap;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // x = lo, y = hi
    return *reinterpret_cast<uint32_t*>(&v);
}

template <class C>
__global__ void __launch_bounds__(kThreads) encode_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                              const __grid_constant__ CUtensorMap wkmap,
                                                              const __grid_constant__ CUtensorMap wvmap,
                                                              EncParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::NST * C::STAGE);
    uint64_t* full = bars;                 // [NST]
    uint64_t* empty = bars + C::NST;       // [NST]
    uint64_t* acc_full = bars + 2 * C::NST;  // [2] an item's accumulators complete
    uint64_t* acc_empty = acc_full + 2;      // [2] read out by the four epilogue warps
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = p.S / kKc;
    // work item it -> (slot = L * Hg + h, tile): slot-major
    auto item = [&](int it, int& tile, int& slot) {
        slot = it / p.ntiles;
        tile = it - slot * p.ntiles;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(acc_full + i, 1);
            mbar_init(acc_empty + i, 4);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        if (elect_one()) {
            prefetch_tensormap(&xmap);
            prefetch_tensormap(&wkmap);
            prefetch_tensormap(&wvmap);
            const uint64_t pol_x = policy_evict_first(), pol_w = policy_evict_last();
            int issued = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x) {
                int tile, slot;
                item(it, tile, slot);
                const int L = slot / p.Hg, h = slot - L * p.Hg;
                const int layer = p.layer_begin + L;
                const int wrow_k = (layer * p.Hg + h) * C::RK, wrow_v = (layer * p.Hg + h) * C::RV;
                for (int kc = 0; kc < nk; ++kc) {
                    const int s = issued % C::NST, round = issued / C::NST;
                    if (round > 0 && !(ok = mbar_wait(empty + s, (round - 1) & 1, p.status, 4u, 20))) break;
                    uint8_t* st = smem + size_t(s) * C::STAGE;
                    mbar_expect_tx(full + s, C::STAGE);
                    // x: dims (S, slot = (L*Hg + h)*2 + axis, token): one box per axis
                    for (int axis = 0; axis < 2; ++axis)
                        asm volatile(
                            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
                            " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(st + axis * C::A_BYTES)),
                            "l"(reinterpret_cast<uint64_t>(&xmap)), "r"(kc * kKc), "r"(slot * 2 + axis),
                            "r"(tile * kTok), "r"(smem_u32(full + s)), "l"(pol_x)
                            : "memory");
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
                        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(st + 2 * C::A_BYTES)),
                        "l"(reinterpret_cast<uint64_t>(&wkmap)), "r"(kc * kKc), "r"(wrow_k), "r"(smem_u32(full + s)),
                        "l"(pol_w)
                        : "memory");
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
                        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(st + 2 * C::A_BYTES + C::BK_BYTES)),
                        "l"(reinterpret_cast<uint64_t>(&wvmap)), "r"(kc * kKc), "r"(wrow_v), "r"(smem_u32(full + s)),
                        "l"(pol_w)
                        : "memory");
                    ++issued;
                }
            }
            // drain: no copy in flight at exit
            for (int s = 0; s < C::NST && s < issued; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % C::NST);
                mbar_wait(full + s, (last / C::NST) & 1, p.status, 4u, 21);
            }
        }
    } else if (warp == 1) {
        if (elect_one()) {
            bool ok = true;
            int consumed = 0, j = 0;
            for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x, ++j) {
                const int buf = j & 1, use = j >> 1;
                if (use > 0 && !(ok = mbar_wait(acc_empty + buf, (use - 1) & 1, p.status, 4u, 25))) break;
                tc_fence_after();
                const uint32_t dk = tmem + buf * C::ACC_COLS, dv = dk + C::VCOL;
                for (int kc = 0; kc < nk; ++kc) {
                    const int s = consumed % C::NST, round = consumed / C::NST;
                    if (!(ok = mbar_wait(full + s, round & 1, p.status, 4u, 22))) break;
                    tc_fence_after();
                    const uint32_t ak = smem_u32(smem + size_t(s) * C::STAGE), av = ak + C::A_BYTES;
                    const uint32_t bk = av + C::A_BYTES, bv = bk + C::BK_BYTES;
#pragma unroll
                    for (int kk = 0; kk < kKc / 16; ++kk) {
                        const uint32_t acc = (kc > 0 || kk > 0) ? 1u : 0u;
                        mma_f16_ss(dk, sw128_kmajor_desc(ak + kk * 32), sw128_kmajor_desc(bk + kk * 32), C::IDESC_K, acc);
                        mma_f16_ss(dv, sw128_kmajor_desc(av + kk * 32), sw128_kmajor_desc(bv + kk * 32), C::IDESC_V, acc);
                    }
                    mma_commit(empty + s);
                    ++consumed;
                }
                if (ok) mma_commit(acc_full + buf);
            }
        }
    } else {
        // epilogue: warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
        const int qd = warp & 3;
        const int r = 32 * qd + lane;
        bool ok = true;
        int j = 0;
        for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x, ++j) {
            int tile, slot;
            item(it, tile, slot);
            const int L = slot / p.Hg, h = slot - L * p.Hg;
            const int layer = p.layer_begin + L;
            const int i = tile * kTok + r;
            // the row's destination, read before the accumulators are ready
            int sq = -1, tk = -1;
            if (i < p.n) {
                sq = __ldg(p.seq_idx + i);
                tk = __ldg(p.tok_idx + i);
            }
            const int buf = j & 1, use = j >> 1;
            ok = __all_sync(0xffffffffu, mbar_wait(acc_full + buf, use & 1, p.status, 4u, 24));
            if (!ok) break;
            tc_fence_after();
            const uint32_t taddr = tmem + buf * C::ACC_COLS + (uint32_t(32 * qd) << 16);
            bool write = i < p.n && sq >= 0 && sq < p.batch && tk >= 0 && tk < p.max_tokens;
            const long long ri = write ? p.smap.row_index(sq, layer, tk, p.D, p.max_tokens) : 0;
            write = write && ri >= 0;  // a page index out of range: not written
            uint16_t* dst = p.store + size_t(ri < 0 ? 0 : ri) * p.row + size_t(h) * (C::RK + C::RV);
            const float* bk = p.bias_k + (size_t(layer) * p.Hg + h) * C::RK;
            const float* bv = p.bias_v + (size_t(layer) * p.Hg + h) * C::RV;
#pragma unroll
            for (int a0 = 0; a0 < C::RK; a0 += 16) {
                float v[16];
                tmem_ld<16>(taddr + a0, v);
                tmem_wait_ld();
                if (write) {
                    uint4 w0, w1;
                    w0.x = pack_bf16(v[0] - bk[a0 + 0], v[1] - bk[a0 + 1]);
                    w0.y = pack_bf16(v[2] - bk[a0 + 2], v[3] - bk[a0 + 3]);
                    w0.z = pack_bf16(v[4] - bk[a0 + 4], v[5] - bk[a0 + 5]);
                    w0.w = pack_bf16(v[6] - bk[a0 + 6], v[7] - bk[a0 + 7]);
                    w1.x = pack_bf16(v[8] - bk[a0 + 8], v[9] - bk[a0 + 9]);
                    w1.y = pack_bf16(v[10] - bk[a0 + 10], v[11] - bk[a0 + 11]);
                    w1.z = pack_bf16(v[12] - bk[a0 + 12], v[13] - bk[a0 + 13]);
                    w1.w = pack_bf16(v[14] - bk[a0 + 14], v[15] - bk[a0 + 15]);
                    reinterpret_cast<uint4*>(dst + a0)[0] = w0;
                    reinterpret_cast<uint4*>(dst + a0)[1] = w1;
                }
            }
#pragma unroll
            for (int a0 = 0; a0 < C::RV; a0 += 16) {
                float v[16];
                tmem_ld<16>(taddr + C::VCOL + a0, v);
                tmem_wait_ld();
                if (write) {
                    uint4 w0, w1;
                    w0.x = pack_bf16(v[0] - bv[a0 + 0], v[1] - bv[a0 + 1]);
                    w0.y = pack_bf16(v[2] - bv[a0 + 2], v[3] - bv[a0 + 3]);
                    w0.z = pack_bf16(v[4] - bv[a0 + 4], v[5] - bv[a0 + 5]);
                    w0.w = pack_bf16(v[6] - bv[a0 + 6], v[7] - bv[a0 + 7]);
                    w1.x = pack_bf16(v[8] - bv[a0 + 8], v[9] - bv[a0 + 9]);
                    w1.y = pack_bf16(v[10] - bv[a0 + 10], v[11] - bv[a0 + 11]);
                    w1.z = pack_bf16(v[12] - bv[a0 + 12], v[13] - bv[a0 + 13]);
                    w1.w = pack_bf16(v[14] - bv[a0 + 14], v[15] - bv[a0 + 15]);
                    reinterpret_cast<uint4*>(dst + C::RK + a0)[0] = w0;
                    reinterpret_cast<uint4*>(dst + C::RK + a0)[1] = w1;
                }
            }
            // this warp's lanes of the buffer are read: the MMAs of the item after next may use it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty + buf);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Wide codecs (r_k + r_v = 256): one CTA per SM, and a 64-element chunk of W_down for both axes is
// as large as the stacks of 128 tokens, so half of a 128-token ring would hold L2-resident weights.
// Here a work item is 256 tokens and runs as two phases, the K axis then the V axis: a stage holds
// one axis' stacks of the 256 tokens and that axis' W_down chunk, which serves both 128-token
// halves (two M = 128 MMAs on one B operand).  TMEM holds the K accumulators of both halves
// (2 r_k columns) and the V accumulators (2 r_v columns): the epilogue drains K while the MMAs of
// V run, and V while those of the next item's K run.
constexpr int kTokW = 256;

template <int RK_, int RV_>
struct WCfg {
    static constexpr int RK = RK_, RV = RV_;
    static constexpr int TOK = kTokW;  // tokens per work item
    static constexpr int CTAS_PER_SM = 1;
    static constexpr bool WIDE = true;
    static constexpr int A_BYTES = kTokW * kKc * 2;  // one axis' stacks of the 256 tokens, 64 K elements
    static constexpr int HALF = kTok * kKc * 2;      // offset of the second 128-token half
    static constexpr int BK_BYTES = RK * kKc * 2;
    static constexpr int BV_BYTES = RV * kKc * 2;
    static constexpr int STAGE = A_BYTES + (BK_BYTES > BV_BYTES ? BK_BYTES : BV_BYTES);  // [A | W of the axis]
    static constexpr int NST_FIT = (kSmemLimit - 2048) / STAGE;
    static constexpr int NST = NST_FIT > 6 ? 6 : NST_FIT;
    static constexpr int SMEM = 1024 + NST * STAGE + 1024;
    static constexpr int VCOL = (2 * RK + 15) / 16 * 16;  // TMEM: K of both halves, then V of both
    static constexpr int TMEM_COLS = 512;
    static constexpr uint32_t IDESC_K = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(RK >> 3) << 17) | (uint32_t(128 >> 4) << 24);
    static constexpr uint32_t IDESC_V = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(RV >> 3) << 17) | (uint32_t(128 >> 4) << 24);
    static_assert(RK % 16 == 0 && RV % 16 == 0 && RK <= 256 && RV <= 256, "ranks");
    static_assert(VCOL + 2 * RV <= TMEM_COLS, "TMEM");
    static_assert(STAGE % 1024 == 0 && HALF % 1024 == 0, "swizzle atoms");
    static_assert(NST >= 3 && SMEM <= kSmemLimit && SMEM > kSmemLimit / 2, "one CTA per SM");
};

// Subtract the bias from R accumulator columns of this thread's TMEM lane, round to bf16 and store.
template <int R>
__device__ __forceinline__ void drain_row(uint32_t taddr, uint16_t* dst, const float* bias, bool write) {
#pragma unroll
    for (int a0 = 0; a0 < R; a0 += 16) {
        float v[16];
        tmem_ld<16>(taddr + a0, v);
        tmem_wait_ld();
        if (write) {
            uint4 w0, w1;
            w0.x = pack_bf16(v[0] - bias[a0 + 0], v[1] - bias[a0 + 1]);
            w0.y = pack_bf16(v[2] - bias[a0 + 2], v[3] - bias[a0 + 3]);
            w0.z = pack_bf16(v[4] - bias[a0 + 4], v[5] - bias[a0 + 5]);
            w0.w = pack_bf16(v[6] - bias[a0 + 6], v[7] - bias[a0 + 7]);
            w1.x = pack_bf16(v[8] - bias[a0 + 8], v[9] - bias[a0 + 9]);
            w1.y = pack_bf16(v[10] - bias[a0 + 10], v[11] - bias[a0 + 11]);
            w1.z = pack_bf16(v[12] - bias[a0 + 12], v[13] - bias[a0 + 13]);
            w1.w = pack_bf16(v[14] - bias[a0 + 14], v[15] - bias[a0 + 15]);
            reinterpret_cast<uint4*>(dst + a0)[0] = w0;
            reinterpret_cast<uint4*>(dst + a0)[1] = w1;
        }
    }
}

template <class C>
__global__ void __launch_bounds__(kThreads) encode_tc_wide_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                   const __grid_constant__ CUtensorMap wkmap,
                                                                   const __grid_constant__ CUtensorMap wvmap,
                                                                   EncParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::NST * C::STAGE);
    uint64_t* full = bars;                     // [NST]
    uint64_t* empty = bars + C::NST;           // [NST]
    uint64_t* acc_full = bars + 2 * C::NST;    // [axis] a phase's accumulators complete
    uint64_t* acc_empty = acc_full + 2;        // [axis] read out by the four epilogue warps
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = p.S / kKc;
    auto item = [&](int it, int& tile, int& slot) {  // slot-major, as in the 128-token kernel
        slot = it / p.ntiles;
        tile = it - slot * p.ntiles;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(acc_full + i, 1);
            mbar_init(acc_empty + i, 4);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        if (elect_one()) {
            prefetch_tensormap(&xmap);
            prefetch_tensormap(&wkmap);
            prefetch_tensormap(&wvmap);
            // stacks at normal L2 priority: the 256-byte promotion of a 128-byte row brings the
            // token's next chunk, which the stage after next reads (evict-first measured 2.5% slower)
            const uint64_t pol_x = policy_evict_normal(), pol_w = policy_evict_last();
            int issued = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x) {
                int tile, slot;
                item(it, tile, slot);
                const int L = slot / p.Hg, h = slot - L * p.Hg;
                const int layer = p.layer_begin + L;
                for (int axis = 0; axis < 2 && ok; ++axis) {
                    const CUtensorMap* wmap = axis ? &wvmap : &wkmap;
                    const int wrow = (layer * p.Hg + h) * (axis ? C::RV : C::RK);
                    const int bytes = C::A_BYTES + (axis ? C::BV_BYTES : C::BK_BYTES);
                    for (int kc = 0; kc < nk; ++kc) {
                        const int s = issued % C::NST, round = issued / C::NST;
                        if (round > 0 && !(ok = mbar_wait(empty + s, (round - 1) & 1, p.status, 4u, 26))) break;
                        uint8_t* st = smem + size_t(s) * C::STAGE;
                        mbar_expect_tx(full + s, bytes);
                        // x: dims (S, slot = (L*Hg + h)*2 + axis, token), 256 token rows
                        asm volatile(
                            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
                            " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(st)),
                            "l"(reinterpret_cast<uint64_t>(&xmap)), "r"(kc * kKc), "r"(slot * 2 + axis),
                            "r"(tile * kTokW), "r"(smem_u32(full + s)), "l"(pol_x)
                            : "memory");
                        asm volatile(
                            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
                            " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(st + C::A_BYTES)),
                            "l"(reinterpret_cast<uint64_t>(wmap)), "r"(kc * kKc), "r"(wrow), "r"(smem_u32(full + s)),
                            "l"(pol_w)
                            : "memory");
                        ++issued;
                    }
                }
            }
            for (int s = 0; s < C::NST && s < issued; ++s) {  // drain: no copy in flight at exit
                const int last = issued - 1 - ((issued - 1 - s) % C::NST);
                mbar_wait(full + s, (last / C::NST) & 1, p.status, 4u, 27);
            }
        }
    } else if (warp == 1) {
        if (elect_one()) {
            bool ok = true;
            int consumed = 0, j = 0;
            for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x, ++j) {
                for (int axis = 0; axis < 2 && ok; ++axis) {
                    if (j > 0 && !(ok = mbar_wait(acc_empty + axis, (j - 1) & 1, p.status, 4u, 28))) break;
                    tc_fence_after();
                    const uint32_t d0 = tmem + (axis ? C::VCOL : 0), d1 = d0 + (axis ? C::RV : C::RK);
                    const uint32_t idesc = axis ? C::IDESC_V : C::IDESC_K;
                    for (int kc = 0; kc < nk; ++kc) {
                        const int s = consumed % C::NST, round = consumed / C::NST;
                        if (!(ok = mbar_wait(full + s, round & 1, p.status, 4u, 29))) break;
                        tc_fence_after();
                        const uint32_t a = smem_u32(smem + size_t(s) * C::STAGE), b = a + C::A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < kKc / 16; ++kk) {
                            const uint32_t acc = (kc > 0 || kk > 0) ? 1u : 0u;
                            const uint64_t bd = sw128_kmajor_desc(b + kk * 32);
                            mma_f16_ss(d0, sw128_kmajor_desc(a + kk * 32), bd, idesc, acc);
                            mma_f16_ss(d1, sw128_kmajor_desc(a + C::HALF + kk * 32), bd, idesc, acc);
                        }
                        mma_commit(empty + s);
                        ++consumed;
                    }
                    if (ok) mma_commit(acc_full + axis);
                }
            }
        }
    } else {
        // epilogue: warps 2..5 -> TMEM lane quarters 2, 3, 0, 1; a thread owns one token of each half
        const int qd = warp & 3;
        const int r = 32 * qd + lane;
        bool ok = true;
        int j = 0;
        for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x, ++j) {
            int tile, slot;
            item(it, tile, slot);
            const int L = slot / p.Hg, h = slot - L * p.Hg;
            const int layer = p.layer_begin + L;
            uint16_t* dst[2];
            bool write[2];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {  // the rows' destinations, read before the accumulators are ready
                const int i = tile * kTokW + hf * kTok + r;
                int sq = -1, tk = -1;
                if (i < p.n) {
                    sq = __ldg(p.seq_idx + i);
                    tk = __ldg(p.tok_idx + i);
                }
                bool w = i < p.n && sq >= 0 && sq < p.batch && tk >= 0 && tk < p.max_tokens;
                const long long ri = w ? p.smap.row_index(sq, layer, tk, p.D, p.max_tokens) : 0;
                write[hf] = w && ri >= 0;  // a page index out of range: not written
                dst[hf] = p.store + size_t(ri < 0 ? 0 : ri) * p.row + size_t(h) * (C::RK + C::RV);
            }
            const float* bk = p.bias_k + (size_t(layer) * p.Hg + h) * C::RK;
            const float* bv = p.bias_v + (size_t(layer) * p.Hg + h) * C::RV;
            const uint32_t lanes = uint32_t(32 * qd) << 16;
            for (int axis = 0; axis < 2; ++axis) {
                ok = __all_sync(0xffffffffu, mbar_wait(acc_full + axis, j & 1, p.status, 4u, 30));
                if (!ok) break;
                tc_fence_after();
                if (axis == 0) {
                    drain_row<C::RK>(tmem + lanes, dst[0], bk, write[0]);
                    drain_row<C::RK>(tmem + lanes + C::RK, dst[1], bk, write[1]);
                } else {
                    drain_row<C::RV>(tmem + lanes + C::VCOL, dst[0] + C::RK, bv, write[0]);
                    drain_row<C::RV>(tmem + lanes + C::VCOL + C::RV, dst[1] + C::RK, bv, write[1]);
                }
                // this warp's lanes of the phase's accumulators are read: the next item's MMAs may use them
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty + axis);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

bool make_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
    cuuint32_t es[3] = {1u, 1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class C>
lla_status run_encode(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                      const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* store, int batch, int max_tokens,
                      cudaStream_t stream, const lla_store_map& smap) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return LLA_ERR_CUDA;
    const lla_codec_desc& ds = c->desc;
    const int Hg = ds.variant == 0 ? ds.H : 1;
    const int S = c->S;
    CUtensorMap xmap, wkmap, wvmap;
    {
        cuuint64_t dims[3] = {cuuint64_t(S), cuuint64_t(num_layers) * Hg * 2, cuuint64_t(n)};
        cuuint64_t strides[2] = {cuuint64_t(S) * 2, cuuint64_t(num_layers) * Hg * 2 * S * 2};
        cuuint32_t box[3] = {uint32_t(kKc), 1u, uint32_t(C::TOK)};
        if (!make_map(enc, &xmap, x, 3, dims, strides, box)) return LLA_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {cuuint64_t(S), cuuint64_t(ds.D) * Hg * C::RK};
        cuuint64_t strides[1] = {cuuint64_t(S) * 2};
        cuuint32_t box[2] = {uint32_t(kKc), uint32_t(C::RK)};
        if (!make_map(enc, &wkmap, c->w_down_k_t, 2, dims, strides, box)) return LLA_ERR_CUDA;
    }
    {
        cuuint64_t dims[2] = {cuuint64_t(S), cuuint64_t(ds.D) * Hg * C::RV};
        cuuint64_t strides[1] = {cuuint64_t(S) * 2};
        cuuint32_t box[2] = {uint32_t(kKc), uint32_t(C::RV)};
        if (!make_map(enc, &wvmap, c->w_down_v_t, 2, dims, strides, box)) return LLA_ERR_CUDA;
    }
    EncParams p;
    p.seq_idx = seq_idx;
    p.tok_idx = tok_idx;
    p.store = store;
    p.bias_k = c->bias_k;
    p.bias_v = c->bias_v;
    p.status = c->status;
    p.n = n;
    p.layer_begin = layer_begin;
    p.num_layers = num_layers;
    p.Hg = Hg;
    p.S = S;
    p.D = ds.D;
    p.batch = batch;
    p.max_tokens = max_tokens;
    p.row = size_t(ds.r_k + ds.r_v) * Hg;
    p.smap = smap;
    p.ntiles = (n + C::TOK - 1) / C::TOK;
    const long long items = (long long)p.ntiles * num_layers * Hg;
    if (items > 0x7fffffffLL) return LLA_ERR_UNSUPPORTED_SHAPE;
    p.nitems = int(items);
    void (*kernel)(const CUtensorMap, const CUtensorMap, const CUtensorMap, EncParams);
    if constexpr (C::WIDE)
        kernel = encode_tc_wide_kernel<C>;
    else
        kernel = encode_tc_kernel<C>;
    LLA_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    const long long slots = (long long)lla_num_sms() * C::CTAS_PER_SM;
    const int grid = int(items < slots ? items : slots);
    kernel<<<grid, kThreads, C::SMEM, stream>>>(xmap, wkmap, wvmap, p);
    LLA_CUDA_TRY(cudaGetLastError());
    return LLA_OK;
}

}  // namespace

// Tensor-core encode for the codec shapes it is built for; LLA_ERR_UNSUPPORTED_SHAPE otherwise.
lla_status lla_encode_tc(const lla_codec* c, const uint16_t* x, int n, int layer_begin, int num_layers,
                         const int32_t* seq_idx, const int32_t* tok_idx, uint16_t* store, int batch, int max_tokens,
                         cudaStream_t stream, const lla_store_map& smap) {
    const lla_codec_desc& d = c->desc;
    if (c->S % kKc != 0 || !c->status) return LLA_ERR_UNSUPPORTED_SHAPE;
    if (d.r_k == 16 && d.r_v == 32)
        return run_encode<ECfg<16, 32>>(c, x, n, layer_begin, num_layers, seq_idx, tok_idx, store, batch, max_tokens,
                                        stream, smap);
    if (d.r_k == 96 && d.r_v == 160)
        return run_encode<WCfg<96, 160>>(c, x, n, layer_begin, num_layers, seq_idx, tok_idx, store, batch,
                                         max_tokens, stream, smap);
    if (d.r_k == 64 && d.r_v == 128)
        return run_encode<ECfg<64, 128>>(c, x, n, layer_begin, num_layers, seq_idx, tok_idx, store, batch,
                                         max_tokens, stream, smap);
    return LLA_ERR_UNSUPPORTED_SHAPE;
}
