// The fast path's cache: reconstruct every cached token's loop-t key and value once from the
// latent store and keep them, keys already rotated at their positions.
//
// [LLA summary, "Serving Capacity"]: besides decoding straight from the latent store, a server
// can reconstruct the full K/V once and cache it.  [LLA §3 eq. (3)] gives the rows,
//   k_hat_j = RoPE_j(c^K_j W^K_up,t^T + mu^K_t),   v_hat_j = c^V_j W^V_up,t^T + mu^V_t,
// with RoPE applied after reconstruction [LLA §3, "RoPE and reconstruction"].  The output is the
// head-major bf16 layout lla_full_decode_attn reads: sequence b's head h, token j at element
// b * seq_stride + (h * cache_tokens + j) * d_head.
//
// Tensor-core kernel (d_head 128 and the codec shapes the decode kernels cover): persistent CTAs
// over items (sequence, 128-token tile, head).  Per item the tile's latents are the A operand and
// W_up,t of the head the B operand of tcgen05.mma, K = the latent rank, N = d_head, bf16 in,
// fp32 accumulators in TMEM (128 columns for K, 128 for V, two buffers).  A latent axis is
// staged in panels of 64, 32 or 16 elements (128-, 64- or 32-byte swizzle: one TMA box each for
// the tile's rows and for W_up's rows), a ring of panel stages running on across items.  With
// each item the producer also stages the tile's Phi image (fp16 cos | sin of its 128 positions,
// the codec's decode table) and the head's mu_t, so that four epilogue warps (thread = token
// row) add mu, rotate key pairs (i, i + d/2), round to bf16 and write the rows without a global
// load on their path.  (Reading each row's cos/sin and mu from global memory inside the epilogue
// loop measured 1.03 ms per slice at ratio 4, batch 32 x 4096: 0.32 of the copy peak.)  A warp
// gathers 64 outputs of each of its 32 rows in shared memory and writes them as whole 128-byte
// lines, four rows per store instruction: a 16-byte piece of 32 rows per instruction kept the
// write requests, not DRAM, the limit (0.577 ms per slice against 0.248 ms with the stores
// left out).
//   warp 0  TMA producer   warp 1  TMEM allocator + MMA issuer   warps 2-5  epilogue
// W_up enters the GEMM as bf16 (a copy the codec keeps) and the rotation uses fp16 cos/sin: the
// cache itself is bf16, and both roundings are of the same order as the cache's own or below.
//
// CUDA-core kernel (every other shape): one CTA per (32-token block, head, sequence), the same
// arithmetic in fp32 with W_up in fp32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "lla_internal.cuh"
#include "sm100.cuh"

namespace {

using namespace sm100;

constexpr int kTok = 128;
constexpr int kThreads = 192;
constexpr int kSmemLimit = 232448;
constexpr int kDh = 128;  // d_head of the tensor-core kernel (N of its GEMMs)
constexpr uint32_t kFlagTimeout = 4u;

// Panels of an axis of rank r: 64-element panels first, then at most one of 32 and one of 16.
__host__ __device__ constexpr int num_panels(int r) { return r / 64 + (r % 64) / 32 + (r % 32) / 16; }
__host__ __device__ constexpr int panel_width(int r, int i) {
    return i < r / 64 ? 64 : (i == r / 64 && (r % 64) >= 32) ? 32 : 16;
}
__host__ __device__ constexpr int panel_offset(int r, int i) {
    return i <= r / 64 ? 64 * i : 64 * (r / 64) + 32 * ((r % 64) / 32);
}
// width class: 0 = 64 elements (128-byte swizzle), 1 = 32 (64-byte), 2 = 16 (32-byte)
__host__ __device__ constexpr int width_class(int w) { return w == 64 ? 0 : w == 32 ? 1 : 2; }

template <int RK_, int RV_>
struct RCfg {
    static constexpr int RK = RK_, RV = RV_;
    static constexpr int NPK = num_panels(RK), NPV = num_panels(RV), NP = NPK + NPV;
    static constexpr int A_BYTES = kTok * 64 * 2;   // room for a 64-element panel of the tile's rows
    static constexpr int B_BYTES = kDh * 64 * 2;    // and of W_up's d_head rows
    static constexpr int STAGE = A_BYTES + B_BYTES;
    // per item: the tile's Phi image (fp16 cos | sin of its 128 positions) and the head's mu_t
    static constexpr int PHI_BYTES = kTok * kDh * 2;
    static constexpr int AUX_BYTES = PHI_BYTES + 2 * kDh * 4;
    static constexpr int NST = 4;
    // per epilogue warp: 32 rows x 128 bytes, where a half-row of output is gathered so that the
    // warp writes whole 128-byte lines (four rows per store instruction) instead of one 16-byte
    // piece of each of 32 rows
    static constexpr int XPOSE_BYTES = 4 * 32 * 128;
    static constexpr int SMEM = 1024 + NST * STAGE + 2 * AUX_BYTES + XPOSE_BYTES + 1024;
    static constexpr int ACC_COLS = 2 * kDh;         // K then V accumulator
    static constexpr int TMEM_COLS = 2 * ACC_COLS;   // two buffers
    static constexpr uint32_t IDESC = idesc_bf16_f32(128, kDh, false, false);
    static_assert(RK % 16 == 0 && RV % 16 == 0, "ranks: multiples of 16");
    static_assert(panel_offset(RK, num_panels(RK) - 1) + panel_width(RK, num_panels(RK) - 1) == RK,
                  "K panels cover r_k");
    static_assert(panel_offset(RV, num_panels(RV) - 1) + panel_width(RV, num_panels(RV) - 1) == RV,
                  "V panels cover r_v");
    static_assert(TMEM_COLS <= 512 && NST >= 2 && SMEM <= kSmemLimit, "resources");
};

// tensor maps: A over the layer's latents per width class; B over W_up's bf16 copy per (axis, class)
struct RMaps {
    CUtensorMap a[3];
    CUtensorMap b[2][3];
};

struct RParams {
    const int32_t* seq_lens;
    const uint16_t* phi_tiles;  // codec Phi table: per 128 positions, the fp16 [cos | sin] image
    const float* mu_k;      // codec mu (per-head [D][H][S], 2D [D][S])
    const float* mu_v;
    uint16_t* k_cache;
    uint16_t* v_cache;
    uint32_t* status;
    long long seq_stride;
    int cache_tokens, batch, max_tokens, H, T, S, layer, loop, variant, ntiles, nitems;
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr, int w) {
    // K-major operand, rows of w 16-bit elements in the matching swizzle, 8-row groups 8 rows apart
    const uint32_t row_bytes = uint32_t(w) * 2;
    uint64_t d = 0;
    d |= uint64_t((addr >> 4) & 0x3FFF);
    d |= uint64_t(1) << 16;  // leading byte offset: unused for swizzled K-major
    d |= uint64_t(((8 * row_bytes) >> 4) & 0x3FFF) << 32;
    d |= uint64_t(1) << 46;
    d |= uint64_t(w == 64 ? 2 : w == 32 ? 4 : 6) << 61;  // 128-, 64- or 32-byte swizzle
    return d;
}

// entries k0 .. k0 + 15 of row r of a Phi image (fp16, [k / 64][128 rows][k % 64] with the
// 128-byte swizzle), as floats
__device__ __forceinline__ void phi16(float* v, const uint8_t* img, int r, int k0) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(img + sw128_offset(r, k0 + 8 * c, kTok));
        const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h2[e]);
            v[8 * c + 2 * e] = f.x;
            v[8 * c + 2 * e + 1] = f.y;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// item it -> (sequence b, tile, head h), head fastest; false if the tile holds no cached token
__device__ __forceinline__ bool item_of(const RParams& p, int it, int& b, int& tile, int& h, int& len) {
    h = it % p.H;
    const int bt = it / p.H;
    tile = bt % p.ntiles;
    b = bt / p.ntiles;
    len = __ldg(p.seq_lens + b);
    len = len < 0 ? 0 : (len > p.max_tokens ? p.max_tokens : len);
    return tile * kTok < len;
}

template <class C>
__global__ void __launch_bounds__(kThreads, 1) reconstruct_tc_kernel(const __grid_constant__ RMaps maps, RParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* aux_s = smem + C::NST * C::STAGE;  // [2 items][Phi image | mu^K_t | mu^V_t]
    uint8_t* xpose_s = aux_s + 2 * C::AUX_BYTES;  // [4 epilogue warps][32 rows][128 B]
    uint64_t* bars = reinterpret_cast<uint64_t*>(xpose_s + C::XPOSE_BYTES);
    uint64_t* full = bars;                     // [NST]
    uint64_t* empty = bars + C::NST;           // [NST]
    uint64_t* acc_full = bars + 2 * C::NST;    // [2]
    uint64_t* acc_empty = acc_full + 2;        // [2] read by the four epilogue warps
    uint64_t* aux_full = acc_empty + 2;        // [2]
    uint64_t* aux_empty = aux_full + 2;        // [2]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(aux_empty + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(acc_full + i, 1);
            mbar_init(acc_empty + i, 4);
            mbar_init(aux_full + i, 1);
            mbar_init(aux_empty + i, 4);
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
    // mu_t of head h (d_head floats, 16-byte aligned)
    auto mu_row = [&](const float* mu, int h) {
        return p.variant == 0 ? mu + (size_t(p.layer) * p.H + h) * p.S + size_t(p.loop) * kDh
                              : mu + size_t(p.layer) * p.S + (size_t(p.loop) * p.H + h) * kDh;
    };
    // row of W_up's bf16 copy holding output dimension 0 of (layer, head, loop)
    auto w_row = [&](int h) {
        return p.variant == 0 ? ((p.layer * p.H + h) * p.T + p.loop) * kDh : ((p.layer * p.T + p.loop) * p.H + h) * kDh;
    };

    if (warp == 0) {
        if (elect_one()) {
            const uint64_t pol_lat = policy_evict_first(), pol_w = policy_evict_last();
            int issued = 0, jn = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x) {
                int b, tile, h, len;
                if (!item_of(p, it, b, tile, h, len)) continue;
                const int hmap = p.variant == 0 ? h : 0;
                {
                    const int slot = jn & 1, use = jn >> 1;
                    ++jn;
                    if (use > 0 && !(ok = mbar_wait(aux_empty + slot, (use - 1) & 1, p.status, kFlagTimeout, 85))) break;
                    uint8_t* aux = aux_s + slot * C::AUX_BYTES;
                    mbar_expect_tx(aux_full + slot, C::AUX_BYTES);
                    bulk_g2s(aux, p.phi_tiles + size_t(tile) * (C::PHI_BYTES / 2), C::PHI_BYTES, aux_full + slot, pol_w);
                    bulk_g2s(aux + C::PHI_BYTES, mu_row(p.mu_k, h), kDh * 4, aux_full + slot, pol_w);
                    bulk_g2s(aux + C::PHI_BYTES + kDh * 4, mu_row(p.mu_v, h), kDh * 4, aux_full + slot, pol_w);
                }
                for (int pi = 0; pi < C::NP && ok; ++pi) {
                    const int axis = pi < C::NPK ? 0 : 1;
                    const int r = axis ? C::RV : C::RK, i = axis ? pi - C::NPK : pi;
                    const int w = panel_width(r, i), x = panel_offset(r, i), wc = width_class(w);
                    const int s = issued % C::NST, round = issued / C::NST;
                    if (round > 0 && !(ok = mbar_wait(empty + s, (round - 1) & 1, p.status, kFlagTimeout, 80))) break;
                    uint8_t* st = smem + size_t(s) * C::STAGE;
                    mbar_expect_tx(full + s, uint32_t(w) * 2 * (kTok + kDh));
                    tma_load_4d(st, &maps.a[wc], (axis ? C::RK : 0) + x, hmap, tile * kTok, b, full + s, pol_lat);
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
                        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(st + C::A_BYTES)),
                        "l"(reinterpret_cast<uint64_t>(&maps.b[axis][wc])), "r"(x), "r"(w_row(h)),
                        "r"(smem_u32(full + s)), "l"(pol_w)
                        : "memory");
                    ++issued;
                }
            }
            for (int s = 0; s < C::NST && s < issued; ++s) {  // no copy in flight at exit
                const int last = issued - 1 - ((issued - 1 - s) % C::NST);
                mbar_wait(full + s, (last / C::NST) & 1, p.status, kFlagTimeout, 81);
            }
            for (int s = 0; s < 2 && s < jn; ++s) {
                const int last = jn - 1 - ((jn - 1 - s) % 2);
                mbar_wait(aux_full + s, (last / 2) & 1, p.status, kFlagTimeout, 86);
            }
        }
    } else if (warp == 1) {
        if (elect_one()) {
            bool ok = true;
            int consumed = 0, j = 0;
            for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x) {
                int b, tile, h, len;
                if (!item_of(p, it, b, tile, h, len)) continue;
                const int buf = j & 1, use = j >> 1;
                ++j;
                if (use > 0 && !(ok = mbar_wait(acc_empty + buf, (use - 1) & 1, p.status, kFlagTimeout, 82))) break;
                tc_fence_after();
                for (int pi = 0; pi < C::NP && ok; ++pi) {
                    const int axis = pi < C::NPK ? 0 : 1;
                    const int r = axis ? C::RV : C::RK, i = axis ? pi - C::NPK : pi;
                    const int w = panel_width(r, i);
                    const int s = consumed % C::NST, round = consumed / C::NST;
                    if (!(ok = mbar_wait(full + s, round & 1, p.status, kFlagTimeout, 83))) break;
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + size_t(s) * C::STAGE), bw = a + C::A_BYTES;
                    const uint32_t d = tmem + buf * C::ACC_COLS + axis * kDh;
                    for (int kk = 0; kk < w / 16; ++kk)
                        mma_f16_ss(d, kmajor_desc(a + kk * 32, w), kmajor_desc(bw + kk * 32, w), C::IDESC,
                                   (i > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(empty + s);
                    ++consumed;
                }
                if (ok) mma_commit(acc_full + buf);
            }
        }
    } else {
        // epilogue: warps 2..5 -> TMEM lane quarters 2, 3, 0, 1; thread = token row of the tile
        const int qd = warp & 3, row = 32 * qd + lane;
        // this warp's gather rows: row r's 16-byte chunk c at r * 128 + (c ^ (r % 8)) * 16, so that
        // eight consecutive rows' chunk c fall in eight different bank groups
        uint8_t* xp = xpose_s + (warp - 2) * (32 * 128);
        auto gather = [&](int c, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
            *reinterpret_cast<uint4*>(xp + lane * 128 + ((c ^ (lane & 7)) << 4)) = make_uint4(w0, w1, w2, w3);
        };
        bool ok = true;
        int j = 0;
        for (int it = blockIdx.x; it < p.nitems && ok; it += gridDim.x) {
            int b, tile, h, len;
            if (!item_of(p, it, b, tile, h, len)) continue;
            const int buf = j & 1, use = j >> 1;
            ++j;
            // rows of this warp: tile rows 32 qd .. 32 qd + 31, row r of the tile at
            // rbase + r * d_head (keys and values alike), written only below the sequence length
            const size_t rbase = size_t(b) * p.seq_stride + (size_t(h) * p.cache_tokens + size_t(tile) * kTok) * kDh;
            const int nrows = len - tile * kTok;  // rows of the tile below the length (> 0)
            // the gathered half-row (64 outputs, 128 bytes) of each row, out as whole lines:
            // lane l stores chunk l % 8 of row 4 s + l / 8
            auto flush = [&](uint16_t* cache, int half) {
                __syncwarp();
#pragma unroll
                for (int s4 = 0; s4 < 8; ++s4) {
                    const int r = 4 * s4 + (lane >> 3), c = lane & 7;
                    const uint4 v = *reinterpret_cast<const uint4*>(xp + r * 128 + ((c ^ (r & 7)) << 4));
                    if (32 * qd + r < nrows)
                        *reinterpret_cast<uint4*>(cache + rbase + size_t(32 * qd + r) * kDh + half * 64 + c * 8) = v;
                }
                __syncwarp();
            };
            bool w = mbar_wait(aux_full + buf, use & 1, p.status, kFlagTimeout, 87);
            w = w && mbar_wait(acc_full + buf, use & 1, p.status, kFlagTimeout, 84);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
            tc_fence_after();
            const uint8_t* phi = aux_s + buf * C::AUX_BYTES;
            const float* muk = reinterpret_cast<const float*>(phi + C::PHI_BYTES);
            const float* muv = muk + kDh;
            const uint32_t taddr = tmem + buf * C::ACC_COLS + (uint32_t(32 * qd) << 16);
            // keys: pairs (i, i + 64) rotated by the token's position; cos and sin of the row's
            // position from the Phi image (k < 64: cos, k >= 64: sin; 128-byte swizzle).  The
            // first halves are gathered as they come, the second ones kept in registers until
            // those are out (one CTA per SM: the launch bounds leave room for them)
            uint32_t hi[kDh / 4];
#pragma unroll
            for (int c0 = 0; c0 < kDh / 2; c0 += 16) {
                float x[16], y[16];
                tmem_ld<16>(taddr + c0, x);
                tmem_ld<16>(taddr + c0 + kDh / 2, y);
                float cv[16], sv[16];
                phi16(cv, phi, row, c0);
                phi16(sv, phi, row, c0 + kDh / 2);
                tmem_wait_ld();
                uint32_t lo[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    const float x0 = x[e] + muk[c0 + e], y0 = y[e] + muk[c0 + e + kDh / 2];
                    const float x1 = x[e + 1] + muk[c0 + e + 1], y1 = y[e + 1] + muk[c0 + e + 1 + kDh / 2];
                    lo[e / 2] = pack_bf16x2(x0 * cv[e] - y0 * sv[e], x1 * cv[e + 1] - y1 * sv[e + 1]);
                    hi[c0 / 2 + e / 2] = pack_bf16x2(y0 * cv[e] + x0 * sv[e], y1 * cv[e + 1] + x1 * sv[e + 1]);
                }
                gather(c0 / 8, lo[0], lo[1], lo[2], lo[3]);
                gather(c0 / 8 + 1, lo[4], lo[5], lo[6], lo[7]);
            }
            flush(p.k_cache, 0);
#pragma unroll
            for (int c = 0; c < 8; ++c) gather(c, hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
            flush(p.k_cache, 1);
            // values, one half-row at a time
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int c0 = 0; c0 < kDh / 2; c0 += 16) {
                    const int col = half * (kDh / 2) + c0;
                    float v[16];
                    tmem_ld<16>(taddr + kDh + col, v);
                    tmem_wait_ld();
                    uint32_t o[8];
#pragma unroll
                    for (int e = 0; e < 16; e += 2) o[e / 2] = pack_bf16x2(v[e] + muv[col + e], v[e + 1] + muv[col + e + 1]);
                    gather(c0 / 8, o[0], o[1], o[2], o[3]);
                    gather(c0 / 8 + 1, o[4], o[5], o[6], o[7]);
                }
                flush(p.v_cache, half);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(acc_empty + buf);
                mbar_arrive(aux_empty + buf);
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

// ---------------------------------------------------------------------------------------------
// CUDA-core kernel: any shape.  CTA (32-token block, head, sequence); a thread takes (token,
// pair i) items: x_i and x_{i+d/2} of the key, rotated, and the same two entries of the value.
// ---------------------------------------------------------------------------------------------

struct SParams {
    const uint16_t* store;
    const int32_t* seq_lens;
    const float* w_up_k;  // per-head [D][H][T][d][r_k]; 2D [D][T][H][d][r_k]
    const float* w_up_v;
    const float* mu_k;
    const float* mu_v;
    const float* rope_cos;
    const float* rope_sin;
    uint16_t* k_cache;
    uint16_t* v_cache;
    long long seq_stride;
    int cache_tokens, max_tokens, D, H, T, d, r_k, r_v, S, layer, loop, variant;
};

constexpr int kSimtTok = 32;

__global__ void __launch_bounds__(128) reconstruct_simt_kernel(SParams p) {
    const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    int len = __ldg(p.seq_lens + b);
    len = len < 0 ? 0 : (len > p.max_tokens ? p.max_tokens : len);
    const int t0 = blk * kSimtTok;
    if (t0 >= len) return;
    const int half = p.d / 2, row_elems = p.r_k + p.r_v;
    const size_t slot = p.variant == 0 ? (size_t(p.layer) * p.H + h) * p.T + p.loop
                                       : (size_t(p.layer) * p.T + p.loop) * p.H + h;
    const float* Wk = p.w_up_k + slot * size_t(p.d) * p.r_k;
    const float* Wv = p.w_up_v + slot * size_t(p.d) * p.r_v;
    const float* muk = p.variant == 0 ? p.mu_k + (size_t(p.layer) * p.H + h) * p.S + size_t(p.loop) * p.d
                                      : p.mu_k + size_t(p.layer) * p.S + (size_t(p.loop) * p.H + h) * p.d;
    const float* muv = p.variant == 0 ? p.mu_v + (size_t(p.layer) * p.H + h) * p.S + size_t(p.loop) * p.d
                                      : p.mu_v + size_t(p.layer) * p.S + (size_t(p.loop) * p.H + h) * p.d;
    const int hrow = p.variant == 0 ? p.H : 1, hh = p.variant == 0 ? h : 0;
    const int ntok = min(kSimtTok, len - t0);
    for (int e = threadIdx.x; e < ntok * half; e += blockDim.x) {
        const int j = t0 + e / half, i = e % half;
        const uint16_t* c = p.store + ((size_t(b) * p.D + p.layer) * p.max_tokens + j) * size_t(hrow) * row_elems +
                            size_t(hh) * row_elems;
        float x = muk[i], y = muk[i + half], u = muv[i], v = muv[i + half];
        for (int a = 0; a < p.r_k; ++a) {
            const float ca = bf16_to_f32(c[a]);
            x = fmaf(ca, Wk[size_t(i) * p.r_k + a], x);
            y = fmaf(ca, Wk[size_t(i + half) * p.r_k + a], y);
        }
        for (int a = 0; a < p.r_v; ++a) {
            const float ca = bf16_to_f32(c[p.r_k + a]);
            u = fmaf(ca, Wv[size_t(i) * p.r_v + a], u);
            v = fmaf(ca, Wv[size_t(i + half) * p.r_v + a], v);
        }
        const float cv = p.rope_cos[size_t(j) * half + i], sv = p.rope_sin[size_t(j) * half + i];
        const size_t o = size_t(b) * p.seq_stride + (size_t(h) * p.cache_tokens + j) * p.d;
        const __nv_bfloat16 kx = __float2bfloat16_rn(x * cv - y * sv), ky = __float2bfloat16_rn(y * cv + x * sv);
        p.k_cache[o + i] = *reinterpret_cast<const uint16_t*>(&kx);
        p.k_cache[o + i + half] = *reinterpret_cast<const uint16_t*>(&ky);
        const __nv_bfloat16 vu = __float2bfloat16_rn(u), vv = __float2bfloat16_rn(v);
        p.v_cache[o + i] = *reinterpret_cast<const uint16_t*>(&vu);
        p.v_cache[o + i + half] = *reinterpret_cast<const uint16_t*>(&vv);
    }
}

// ---------------------------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------------------------

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

CUtensorMapSwizzle swizzle_of(int w) {
    return w == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : w == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

template <class C>
lla_status run_tc(const lla_reconstruct_call& rc) {
    const lla_codec* c = rc.codec;
    const lla_codec_desc& ds = c->desc;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return LLA_ERR_CUDA;
    RMaps maps;
    memset(&maps, 0, sizeof(maps));
    const int hmap = ds.variant == 0 ? ds.H : 1;
    const size_t row_bytes = size_t(hmap) * (C::RK + C::RV) * 2;
    const void* base = rc.store + size_t(rc.layer) * rc.max_tokens * (row_bytes / 2);
    for (int wc = 0; wc < 3; ++wc) {
        const int w = wc == 0 ? 64 : wc == 1 ? 32 : 16;
        cuuint64_t dims[4] = {cuuint64_t(C::RK + C::RV), cuuint64_t(hmap), cuuint64_t(rc.max_tokens),
                              cuuint64_t(rc.batch)};
        cuuint64_t strides[3] = {cuuint64_t(C::RK + C::RV) * 2, cuuint64_t(row_bytes),
                                 cuuint64_t(row_bytes) * rc.max_tokens * ds.D};
        cuuint32_t box[4] = {uint32_t(w), 1u, uint32_t(kTok), 1u}, es[4] = {1u, 1u, 1u, 1u};
        if (enc(&maps.a[wc], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(w), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return LLA_ERR_CUDA;
        for (int axis = 0; axis < 2; ++axis) {
            const int r = axis ? C::RV : C::RK;
            if (w > r) continue;  // no panel of this width on this axis
            cuuint64_t bd[2] = {cuuint64_t(r), cuuint64_t(ds.D) * ds.T * ds.H * kDh};
            cuuint64_t bs[1] = {cuuint64_t(r) * 2};
            cuuint32_t bb[2] = {uint32_t(w), uint32_t(kDh)}, be[2] = {1u, 1u};
            if (enc(&maps.b[axis][wc], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    axis ? static_cast<void*>(c->w_up_v_bf16) : static_cast<void*>(c->w_up_k_bf16), bd, bs, bb, be,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_of(w), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                return LLA_ERR_CUDA;
        }
    }
    RParams p;
    p.seq_lens = rc.seq_lens;
    p.phi_tiles = c->phi_tiles;
    p.mu_k = c->mu_k;
    p.mu_v = c->mu_v;
    p.k_cache = rc.k_cache;
    p.v_cache = rc.v_cache;
    p.status = c->status;
    p.seq_stride = rc.seq_stride;
    p.cache_tokens = rc.cache_tokens;
    p.batch = rc.batch;
    p.max_tokens = rc.max_tokens;
    p.H = ds.H;
    p.T = ds.T;
    p.S = c->S;
    p.layer = rc.layer;
    p.loop = rc.loop;
    p.variant = ds.variant;
    p.ntiles = (rc.max_tokens + kTok - 1) / kTok;
    const long long items = (long long)rc.batch * p.ntiles * ds.H;
    if (items > 0x7fffffffLL) return LLA_ERR_UNSUPPORTED_SHAPE;
    p.nitems = int(items);
    if (p.nitems == 0) return LLA_OK;
    LLA_CUDA_TRY(cudaFuncSetAttribute(reconstruct_tc_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    const int grid = p.nitems < lla_num_sms() ? p.nitems : lla_num_sms();
    reconstruct_tc_kernel<C><<<grid, kThreads, C::SMEM, rc.stream>>>(maps, p);
    LLA_CUDA_TRY(cudaGetLastError());
    return LLA_OK;
}

lla_status run_simt(const lla_reconstruct_call& rc) {
    const lla_codec* c = rc.codec;
    const lla_codec_desc& ds = c->desc;
    SParams p;
    p.store = rc.store;
    p.seq_lens = rc.seq_lens;
    p.w_up_k = c->w_up_k;
    p.w_up_v = c->w_up_v;
    p.mu_k = c->mu_k;
    p.mu_v = c->mu_v;
    p.rope_cos = c->rope_cos;
    p.rope_sin = c->rope_sin;
    p.k_cache = rc.k_cache;
    p.v_cache = rc.v_cache;
    p.seq_stride = rc.seq_stride;
    p.cache_tokens = rc.cache_tokens;
    p.max_tokens = rc.max_tokens;
    p.D = ds.D;
    p.H = ds.H;
    p.T = ds.T;
    p.d = ds.d_head;
    p.r_k = ds.r_k;
    p.r_v = ds.r_v;
    p.S = c->S;
    p.layer = rc.layer;
    p.loop = rc.loop;
    p.variant = ds.variant;
    const int blocks = (rc.max_tokens + kSimtTok - 1) / kSimtTok;
    if (blocks == 0) return LLA_OK;
    if (rc.batch > 65535 || ds.H > 65535) return LLA_ERR_UNSUPPORTED_SHAPE;
    reconstruct_simt_kernel<<<dim3(blocks, ds.H, rc.batch), 128, 0, rc.stream>>>(p);
    LLA_CUDA_TRY(cudaGetLastError());
    return LLA_OK;
}

}  // namespace

bool lla_reconstruct_tc_supported(const lla_codec* c) {
    const lla_codec_desc& d = c->desc;
    if (d.d_head != kDh || !c->w_up_k_bf16 || !c->w_up_v_bf16 || !c->phi_tiles) return false;
    if (d.variant == 0) return (d.r_k == 16 && d.r_v == 32) || (d.r_k == 96 && d.r_v == 160);
    return d.r_k == 64 && d.r_v == 128;
}

lla_status lla_reconstruct_launch(const lla_reconstruct_call& rc, int impl) {
    if (impl == 1 || (impl == 0 && !lla_reconstruct_tc_supported(rc.codec))) return run_simt(rc);
    if (!lla_reconstruct_tc_supported(rc.codec)) return LLA_ERR_UNSUPPORTED_SHAPE;
    const lla_codec_desc& d = rc.codec->desc;
    if (d.variant == 1) return run_tc<RCfg<64, 128>>(rc);
    if (d.r_k == 16) return run_tc<RCfg<16, 32>>(rc);
    return run_tc<RCfg<96, 160>>(rc);
}
