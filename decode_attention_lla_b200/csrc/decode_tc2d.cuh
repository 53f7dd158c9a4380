// LLA-2D tensor-core decode kernel for sm_100a (part of the decode_tc.cu translation unit).
//
// [LLA §3, "LLA-2D"]: one latent row (c^K_j | c^V_j) per (sequence, layer, token) serves
// all H heads; the per-(loop, head) up-projections differ.  Scores use the same bilinear
// form as the per-head kernel, G = Phi M_q per group of heads on tcgen05 and an r_k-long
// CUDA-core dot c^K_j . G_j per (token, head).  Because c^V_j is shared by the heads, the
// latent-space V accumulation of [LLA §3 eq. (3)],
//   acc_h += sum_j p_{h,j} c^V_j,
// is itself a GEMM here: per 128-token tile,
//   D [r_v x 16] = (C^V)^T [r_v x 128 tokens] . P [128 tokens x 16]
// with C^V the MN-major operand straight from the TMA stage and P the bf16 probabilities.
// Each 32-token quarter of a tile keeps its own online-softmax state (as in the per-head
// kernel), so the 16 columns are (head of the CTA item, token quarter) and P is block
// diagonal: quarter q's tokens feed only its own columns, and the other entries stay zero.
// The compute warps then rescale and add D into registers: acc_{q,h} = alpha acc_{q,h} + D.
//
// Warp roles (one CTA per SM, persistent over the (head part, sequence, tile) walk):
//   warp 0      TMA: M_q images (per sequence and part), Phi tiles (two buffers), c^K
//               quarter slots (one 128-byte swizzled row per token).
//   warp 1      TMEM allocator and MMA issuer: per tile the score GEMMs of every head
//               group, then the V GEMM of the previous tile (its P is complete by then).
//   warp 2      TMA: c^V quarter slots (two 64-wide swizzled panels per token), the four
//               quarters of a tile on one barrier.
//   warps 3-10  compute: one warp per (TMEM lane quarter, head group of the item; two heads
//               per group).  Per tile: score, softmax, P and alpha into shared memory, then
//               the previous tile's V GEMM result into its accumulators.
// Every wait is bounded and sets a status bit on timeout.

template <int DH_, int RK_, int RV_, int H_>
struct Cfg2 : HeadGroups<DH_, RK_, RV_, H_> {
    using HB = HeadGroups<DH_, RK_, RV_, H_>;
    using HB::DH, HB::RK, HB::RV, HB::H, HB::HG, HB::NG, HB::HC, HB::GPC, HB::MQ_BYTES, HB::MQ_GROUP_BYTES,
        HB::PHI_BYTES;
    static constexpr bool TWO_D = true;
    static constexpr bool WIDE = false;
    static constexpr int ROW = RK + RV;
    static constexpr int QTOK = 32;                     // tokens per TMEM lane quarter
    static constexpr int PANEL = QTOK * 128;            // one 64-wide swizzled panel of a quarter
    static constexpr int K_SLOT = PANEL;                // c^K of a quarter (r_k = 64)
    static constexpr int V_PANELS = RV / 64;
    static constexpr int V_SLOT = V_PANELS * PANEL;     // c^V of a quarter
    static constexpr int NPHI = 2;
    static constexpr int VN = 16;                       // V GEMM columns: (head, quarter)
    static constexpr int P_BYTES = (kTile / 64) * VN * 128;  // [token panel][16 rows][128 B]
    static constexpr int BAR_BYTES = 1024;
    static constexpr int FIXED = 1024 /*align slack*/ + NPHI * PHI_BYTES + MQ_BYTES + 2 * P_BYTES + BAR_BYTES;
    static constexpr int NK = 8;                        // c^K ring: two tiles
    static constexpr int NV_RAW = (kSmemLimit - FIXED - NK * K_SLOT) / V_SLOT;
    static constexpr int NV = NV_RAW > 16 ? 16 : NV_RAW;
    static constexpr int SMEM = FIXED + NK * K_SLOT + NV * V_SLOT;
    static constexpr int HPW = HG;                      // heads per compute warp: one TMEM group
    static constexpr int NCW = 4 * (HC / HPW);          // one compute warp per (quarter, head group)
    static constexpr int THREADS = 32 * (3 + NCW);
    static constexpr int TMEM_COLS = 512;
    static constexpr int NBUF = 3;                      // score accumulator ring
    static constexpr int BUF_COLS = NG;
    static constexpr int VCOL = NBUF * BUF_COLS;        // two V accumulators after the ring
    static constexpr uint32_t IDESC_V = idesc_bf16_f32(128, VN, /*A MN-major*/ true, false);
    static_assert(RK == 64, "c^K quarter slot is one 128-byte row per token");
    static_assert(RV == 128, "the V GEMM has M = r_v = 128");
    static_assert(HC * 4 == VN, "V GEMM columns = heads of the item x quarters");
    static_assert(VCOL + 2 * VN <= TMEM_COLS, "TMEM columns");
    static_assert(NV >= 4, "c^V ring");
    // the c^V producer frees a slot on its tile's d_full phase: the last slot of tile m is refilled
    // at stage 4m + 3 + NV, which must precede tile m + 2's last stage (4m + 11), or d_full[m & 1]
    // could be one phase further on than the parity the producer waits for
    static_assert(NV <= 8, "c^V ring at most two tiles");
    static_assert(SMEM <= kSmemLimit, "shared memory");
    static_assert((6 + 2 * NBUF + 6 + 5 * NK + 4) * 8 + 16 + 2 * 4 * HC * 4 <= BAR_BYTES, "barrier area");
};

// Wait for the last phase of each of `ns` ring barriers after `count` uses in ring order.
__device__ __forceinline__ void wait_last_phases(uint64_t* bars, uint32_t ns, uint32_t count, uint32_t* status,
                                                 uint32_t site) {
    for (uint32_t s = 0; s < ns && s < count; ++s) {
        const uint32_t last = count - 1 - ((count - 1 - s) % ns);
        mbar_wait(bars + s, (last / ns) & 1, status, kFlagTimeout, site);
    }
}

// The same for a ring whose round r of slot s lands on bars[r % 4][s] (four sets of ns).
__device__ __forceinline__ void wait_last_phases4(uint64_t* bars, uint32_t ns, uint32_t count, uint32_t* status,
                                                  uint32_t site) {
    for (uint32_t s = 0; s < ns && s < count; ++s) {
        const uint32_t last = (count - 1 - ((count - 1 - s) % ns)) / ns;  // last round of slot s
        mbar_wait(bars + (last & 3) * ns + s, (last >> 2) & 1, status, kFlagTimeout, site);
    }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) tc2d_decode_kernel(const __grid_constant__ LatMaps maps,
                                                                  TcParams p) {
    const CUtensorMap& lat_map = maps.m[0];
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* phi_s = smem;                               // [NPHI][PHI_BYTES]
    uint8_t* mq_s = phi_s + C::NPHI * C::PHI_BYTES;      // [GPC][MQ_GROUP_BYTES]
    uint8_t* p_s = mq_s + C::MQ_BYTES;                   // [2][P_BYTES]
    uint8_t* k_s = p_s + 2 * C::P_BYTES;                 // [NK][K_SLOT]
    uint8_t* v_s = k_s + C::NK * C::K_SLOT;              // [NV][V_SLOT]
    uint64_t* bars = reinterpret_cast<uint64_t*>(v_s + C::NV * C::V_SLOT);
    uint64_t* phi_full = bars;                // [2]
    uint64_t* phi_empty = bars + 2;           // [2]
    uint64_t* mq_full = bars + 4;
    uint64_t* mq_empty = bars + 5;
    uint64_t* tm_full = bars + 6;             // [NBUF]
    uint64_t* tm_empty = tm_full + C::NBUF;   // [NBUF]
    uint64_t* p_full = tm_empty + C::NBUF;    // [2] P and alpha of a tile written
    uint64_t* d_full = p_full + 2;            // [2] V GEMM of a tile complete
    uint64_t* d_empty = d_full + 2;           // [2] V accumulator read by every compute warp
    // Round r of a ring slot lands on its barrier of set r % 4: compute warps drift apart by up to
    // NBUF head groups, more than a ring round, and with four barriers per slot a parity wait can
    // only alias a round four rounds back, which every reader has long released.
    uint64_t* k_full = d_empty + 2;           // [4][NK]
    uint64_t* k_empty = k_full + 4 * C::NK;
    // c^V of tile n (its four quarter slots) lands on vt_full[n % 4]; a slot is free again once its
    // tile's V GEMM is complete: the producer waits on d_full
    uint64_t* vt_full = k_empty + C::NK;      // [4]
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(vt_full + 4);
    float* alpha_s = reinterpret_cast<float*>(tmem_holder + 4);  // [2][4 quarters][HC]
    auto kf = [&](uint32_t slot, uint32_t round) { return k_full + (round & 3) * C::NK + slot; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // P starts all zero: each compute warp only ever writes its own block of it
    for (int i = threadIdx.x; i < 2 * C::P_BYTES / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(p_s)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(phi_full + i, 1);
            mbar_init(phi_empty + i, 1);
            mbar_init(p_full + i, C::NCW);
            mbar_init(d_full + i, 1);
            mbar_init(d_empty + i, C::NCW);
        }
        mbar_init(mq_full, 1);
        mbar_init(mq_empty, 1);
        for (int i = 0; i < C::NBUF; ++i) {
            mbar_init(tm_full + i, 1);
            mbar_init(tm_empty + i, 4);  // the group's warp of each quarter
        }
        for (int i = 0; i < 4 * C::NK; ++i) mbar_init(k_full + i, 1);
        for (int i = 0; i < C::NK; ++i) mbar_init(k_empty + i, C::HC / C::HPW);  // the group warps of the quarter
        for (int i = 0; i < 4; ++i) mbar_init(vt_full + i, 1);
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

    if (warp == 0) {
        // ------------------------------------------------------------ M_q, Phi, c^K loads
        if (elect_one()) {
            prefetch_tensormap(&lat_map);
            // a latent tile is read by every head part of the group within a short time: plain
            // L2 priority keeps it for them (evict-first let it go before the last part's read)
            const uint64_t pol_stream = policy_evict_normal();
            const uint64_t pol_keep = policy_evict_last();
            uint32_t kk_n = 0, phi_n = 0, mq_n = 0;
            int prev_key = -1;
            bool ok = true;
            for (; wk.valid() && ok; wk.next()) {
                const int key = wk.key();
                if (key != prev_key) {
                    if (mq_n > 0 && !(ok = mbar_wait(mq_empty, (mq_n - 1) & 1, p.status, kFlagTimeout, 21))) break;
                    mbar_expect_tx(mq_full, C::MQ_BYTES);
                    const uint8_t* src = p.mq + (size_t(wk.p) * p.B + wk.b) * C::MQ_BYTES;
                    for (int off = 0; off < C::MQ_BYTES; off += 32768) {
                        const int n = C::MQ_BYTES - off < 32768 ? C::MQ_BYTES - off : 32768;
                        bulk_g2s(mq_s + off, src + off, n, mq_full, pol_keep);
                    }
                    ++mq_n;
                    prev_key = key;
                }
                {
                    const uint32_t pb = phi_n & 1, pr = phi_n >> 1;
                    if (pr > 0 && !(ok = mbar_wait(phi_empty + pb, (pr - 1) & 1, p.status, kFlagTimeout, 22))) break;
                    mbar_expect_tx(phi_full + pb, C::PHI_BYTES);
                    bulk_g2s(phi_s + pb * C::PHI_BYTES, p.phi_tiles + size_t(wk.t) * (C::PHI_BYTES / 2), C::PHI_BYTES,
                             phi_full + pb, pol_keep);
                    ++phi_n;
                }
                int tok, outer;
                tile_coords(p, wk.b, wk.t, tok, outer);
                for (int q = 0; q < 4; ++q) {
                    const uint32_t slot = kk_n % C::NK, round = kk_n / C::NK;
                    if (round > 0 && !(ok = mbar_wait(k_empty + slot, (round - 1) & 1, p.status, kFlagTimeout, 23)))
                        break;
                    mbar_expect_tx(kf(slot, round), C::K_SLOT);
                    tma_load_4d(k_s + size_t(slot) * C::K_SLOT, &lat_map, 0, 0, tok + q * C::QTOK, outer,
                                kf(slot, round), pol_stream);
                    ++kk_n;
                }
            }
            // no copy may still be in flight when the CTA exits
            wait_last_phases4(k_full, C::NK, kk_n, p.status, 24);
            wait_last_phases(phi_full, 2, phi_n, p.status, 25);
            if (mq_n > 0) mbar_wait(mq_full, (mq_n - 1) & 1, p.status, kFlagTimeout, 26);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ c^V loads
        if (elect_one()) {
            const uint64_t pol_stream = policy_evict_normal();
            uint32_t vk_n = 0, vt_n = 0;
            bool ok = true;
            for (; wk.valid() && ok; wk.next(), ++vt_n) {
                int vtok, vouter;
                tile_coords(p, wk.b, wk.t, vtok, vouter);
                // the tile's four quarters on one barrier.  Its previous phase (tile vt_n - 4) is
                // complete: refilling the slots of tile vt_n - 1 needed tile vt_n - 2's V GEMM done
                uint64_t* vbar = vt_full + (vt_n & 3);
                mbar_expect_tx(vbar, 4 * C::V_SLOT);
                for (int q = 0; q < 4; ++q) {
                    const uint32_t slot = vk_n % C::NV, round = vk_n / C::NV;
                    // the slot's previous tile m: its V GEMM complete (d_full[m & 1], phase m / 2).  The
                    // producer never runs two phases ahead: it waited for every earlier tile in order.
                    const uint32_t m = (vk_n - C::NV) / 4;
                    if (round > 0 && !(ok = mbar_wait(d_full + (m & 1), (m >> 1) & 1, p.status, kFlagTimeout, 27)))
                        break;
#pragma unroll
                    for (int pn = 0; pn < C::V_PANELS; ++pn)
                        tma_load_4d(v_s + size_t(slot) * C::V_SLOT + pn * C::PANEL, &lat_map, C::RK + 64 * pn, 0,
                                    vtok + q * C::QTOK, vouter, vbar, pol_stream);
                    ++vk_n;
                }
            }
            // no copy in flight at exit: the last (up to) four tiles' barriers complete.  A tile
            // cut short by a failed wait has bytes that never arrive: its wait gives up (bounded).
            for (uint32_t t = vt_n > 4 ? vt_n - 4 : 0; t < vt_n; ++t)
                mbar_wait(vt_full + (t & 3), (t >> 2) & 1, p.status, kFlagTimeout, 28);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            uint32_t phi_n = 0, mq_n = 0, mq_commits = 0, tile_n = 0, v_next = 0;
            uint32_t v_slot = 0;            // c^V slot of quarter 0 of tile v_next: (4 v_next) % NV
            uint32_t sbuf = 0, suse = 0;    // score buffer of the next head group and its use count
            int prev_key = -1;
            bool ok = true;
            // operand descriptors: built once; an operand's start address moves by adding its byte
            // offset / 16 to the descriptor (the 14-bit address field cannot carry: shared memory
            // addresses stay below 2^18)
            const uint64_t phi_desc = sw128_kmajor_desc(smem_u32(phi_s)), mq_desc = sw128_kmajor_desc(smem_u32(mq_s));
            const uint64_t p_desc = sw128_kmajor_desc(smem_u32(p_s));
            const uint64_t v_desc = sw128_mnmajor_desc(smem_u32(v_s), C::PANEL, 1024);
            // V GEMM of tile n: D[pb] = sum over its 8 sixteen-token steps of (C^V)^T . P
            auto issue_v = [&](uint32_t n) -> bool {
                const uint32_t pb = n & 1, use = n >> 1;
                // p_full also says that the accumulator D[pb] is free: every compute warp waits for
                // d_empty[pb] (its readers of tile n - 2 done) before it writes P of tile n
                if (!mbar_wait(p_full + pb, use & 1, p.status, kFlagTimeout, 29)) return false;
                tc_fence_after();  // the accumulator's readers (tcgen05.ld) are done with it
                const uint32_t d_tmem = tmem_base + C::VCOL + pb * C::VN;
                // TMA-filled operands: the barrier wait alone orders them before the MMA
                if (!mbar_wait(vt_full + (n & 3), (n >> 2) & 1, p.status, kFlagTimeout, 31)) return false;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t slot = v_slot + q < C::NV ? v_slot + q : v_slot + q - C::NV;
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const int kk = 2 * q + k2;  // sixteen-token step of the tile
                        const uint64_t ad = v_desc + ((slot * C::V_SLOT + k2 * (16 * 128)) >> 4);
                        const uint64_t bd = p_desc + ((pb * C::P_BYTES + uint32_t(kk >> 2) * (C::VN * 128) +
                                                       uint32_t(kk & 3) * 32) >> 4);
                        mma_f16_ss(d_tmem, ad, bd, C::IDESC_V, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(d_full + pb);  // also frees the tile's four c^V slots
                v_slot = v_slot + 4 < C::NV ? v_slot + 4 : v_slot + 4 - C::NV;
                return true;
            };
            // V GEMMs of every tile before `end` not issued yet
            auto issue_v_upto = [&](uint32_t end) -> bool {
                for (; v_next < end; ++v_next)
                    if (!issue_v(v_next)) return false;
                return true;
            };
            for (; wk.valid() && ok; wk.next(), ++tile_n) {
                const int key = wk.key();
                if (key != prev_key) {
                    if (prev_key != -1) {
                        mma_commit(mq_empty);
                        ++mq_commits;
                    }
                    // the compute warps close the previous sequence with its last V GEMM: issue
                    // it before waiting for the next M_q image
                    if (!(ok = issue_v_upto(tile_n))) break;
                    if (!(ok = mbar_wait(mq_full, mq_n & 1, p.status, kFlagTimeout, 32))) break;
                    ++mq_n;
                    prev_key = key;
                }
                const uint32_t pb = phi_n & 1;
                if (!(ok = mbar_wait(phi_full + pb, (phi_n >> 1) & 1, p.status, kFlagTimeout, 33))) break;
                ++phi_n;
                const uint64_t phi_d = phi_desc + ((pb * C::PHI_BYTES) >> 4);
                for (int g = 0; g < C::GPC && ok; ++g) {
                    const uint32_t buf = sbuf, use = suse;
                    if (++sbuf == C::NBUF) {
                        sbuf = 0;
                        ++suse;
                    }
                    if (use > 0 && !(ok = mbar_wait(tm_empty + buf, (use - 1) & 1, p.status, kFlagTimeout, 34))) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + buf * C::BUF_COLS;
                    const uint64_t mq_d = mq_desc + ((g * C::MQ_GROUP_BYTES) >> 4);
#pragma unroll
                    for (int kk = 0; kk < C::DH / 16; ++kk) {
                        const uint32_t koff = uint32_t(kk & 3) * 32;
                        const uint64_t ad = phi_d + ((uint32_t(kk >> 2) * (kTile * 128) + koff) >> 4);
                        const uint64_t bd = mq_d + ((uint32_t(kk >> 2) * (C::NG * 128) + koff) >> 4);
                        mma_f16_ss(d_tmem, ad, bd, C::IDESC, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(tm_full + buf);
                }
                if (!ok) break;
                mma_commit(phi_empty + pb);
                ok = issue_v_upto(tile_n);  // the previous tile's P is complete once its scores are
            }
            if (ok) ok = issue_v_upto(tile_n);
            if (prev_key != -1) {
                mma_commit(mq_empty);
                ++mq_commits;
            }
            // the commits' arrivals land in shared memory: see them complete before the CTA exits
            wait_last_phases(phi_empty, 2, phi_n, p.status, 35);
            if (mq_commits > 0) mbar_wait(mq_empty, (mq_commits - 1) & 1, p.status, kFlagTimeout, 37);
        }
    } else {
        // ------------------------------------------------------------ compute warps
        // one warp per (TMEM lane quarter, head group): the HPW heads of a group share the
        // warp's c^K loads and conversions, its waits and its barrier arrivals
        constexpr int HPW = C::HPW;
        const int cw = warp - 3;
        const int qd = warp & 3;            // TMEM lane quarter = token rows [32 qd, 32 qd + 32)
        const int g = cw >> 2;              // head group of the CTA item
        const int hf0 = g * HPW;            // first head of the item in this warp
        const uint32_t lane_addr = uint32_t(32 * qd) << 16;

        float m[HPW], l[HPW], acc[HPW][4], isc[HPW];
        uint32_t p_off[HPW];  // this lane's entry of P, per head
#pragma unroll
        for (int hh = 0; hh < HPW; ++hh) p_off[hh] = sw128_offset((hf0 + hh) * 4 + qd, 32 * qd + lane, C::VN);
        int len = 0;
        uint32_t tile_n = 0;
        int prev_key = -1;
        long long prev_id = 0;
        bool ok = true, pending = false;

        auto sync_ok = [&](bool w) { ok = __all_sync(0xffffffffu, w) && ok; };

        // V GEMM result of tile n: acc_{q,h} = alpha_{q,h} acc_{q,h} + D[:, (h, q)] for the
        // r_v dimensions of this lane quarter, every source quarter q and this warp's heads
        auto accumulate = [&](uint32_t n) {
            const uint32_t pb = n & 1, use = n >> 1;
            // p_full: the alpha values, written before its arrivals; d_full: the GEMM
            bool w = mbar_wait(p_full + pb, use & 1, p.status, kFlagTimeout, 38);
            w = w && mbar_wait(d_full + pb, use & 1, p.status, kFlagTimeout, 39);
            sync_ok(w);
            tc_fence_after();
            float d[4 * HPW];
            tmem_ld<4 * HPW>(tmem_base + lane_addr + C::VCOL + pb * C::VN + hf0 * 4, d);
            tmem_wait_ld();
            const float* al = alpha_s + pb * (4 * C::HC) + hf0;
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[hh][q] = fmaf(acc[hh][q], al[q * C::HC + hh], d[hh * 4 + q]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(d_empty + pb);
        };

        auto flush = [&](long long id) {
            const size_t rl = C::RV + 2;
            float* set = p.records + size_t(id) * 4 * C::HC * rl;  // record (q, h) at (q * HC + h) * rl
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) {
                const int hf = hf0 + hh;
                const float lsum = warp_sum(l[hh]);
                if (lane == 0) {
                    float* own = set + (size_t(qd) * C::HC + hf) * rl;
                    own[0] = (m[hh] == -INFINITY) ? -INFINITY : m[hh] * kLn2;
                    own[1] = lsum;
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) set[(size_t(q) * C::HC + hf) * rl + 2 + 32 * qd + lane] = acc[hh][q];
            }
        };

        for (; wk.valid() && ok; wk.next(), ++tile_n) {
            const int key = wk.key();
            if (key != prev_key) {
                if (pending) {
                    accumulate(tile_n - 1);
                    pending = false;
                }
                if (prev_key != -1) flush(prev_id);
#pragma unroll
                for (int hh = 0; hh < HPW; ++hh) {
                    m[hh] = -INFINITY;
                    l[hh] = 0.f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[hh][q] = 0.f;
                    isc[hh] = __ldg(p.inv_scale + size_t(wk.b) * C::H + wk.p * C::HC + hf0 + hh);
                }
                prev_key = key;
                prev_id = wk.record_id();
                len = __ldg(p.lens + wk.b);
            }
            const int valid = min(kTile, len - wk.t * kTile);
            const int nv = max(0, min(32, valid - 32 * qd));  // valid rows of this quarter
            const bool row_ok = lane < nv;

            // ---- scores of the group's heads: s = c^K . G + bias, G from TMEM
            const uint32_t gi = tile_n * C::GPC + g;
            const uint32_t buf = gi % C::NBUF;
            sync_ok(mbar_wait(tm_full + buf, (gi / C::NBUF) & 1, p.status, kFlagTimeout, 40));
            const uint32_t ks = tile_n * 4 + qd, kslot = ks % C::NK;
            {
                bool w = true;
                if (lane == 0) {
                    w = ok && mbar_wait(kf(kslot, ks / C::NK), (ks / C::NK >> 2) & 1, p.status, kFlagTimeout, 42);
                }
                ok = __shfl_sync(0xffffffffu, w, 0) && ok;
                __syncwarp();
            }
            if (!ok) break;
            tc_fence_after();
            const uint32_t tcol = tmem_base + lane_addr + buf * C::BUF_COLS;
            const uint8_t* krow = k_s + size_t(kslot) * C::K_SLOT + lane * 128;
            float bias[HPW];
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) tmem_ld<1>(tcol + C::HG * C::RK + hh, &bias[hh]);
            uint64_t s01[HPW], s23[HPW];
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) s01[hh] = s23[hh] = 0;
            // 16 latent dimensions at a time, the next 16 columns of G in flight while the
            // current ones are used; the c^K words are converted once for all heads
            float ga[HPW][16], gb[HPW][16];
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) tmem_ld<16>(tcol + hh * C::RK, ga[hh]);
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) tmem_wait_ld_regs16(ga[hh]);
#pragma unroll
            for (int a16 = 0; a16 < C::RK / 16; ++a16) {
                float(*cur)[16] = (a16 & 1) ? gb : ga;
                float(*nxt)[16] = (a16 & 1) ? ga : gb;
                if (a16 + 1 < C::RK / 16) {
#pragma unroll
                    for (int hh = 0; hh < HPW; ++hh) tmem_ld<16>(tcol + hh * C::RK + 16 * (a16 + 1), nxt[hh]);
                }
                const uint4 u0 = *reinterpret_cast<const uint4*>(krow + (((2 * a16) ^ (lane & 7)) << 4));
                const uint4 u1 = *reinterpret_cast<const uint4*>(krow + (((2 * a16 + 1) ^ (lane & 7)) << 4));
                const uint64_t c2[8] = {bf16x2_to_f2(u0.x), bf16x2_to_f2(u0.y), bf16x2_to_f2(u0.z), bf16x2_to_f2(u0.w),
                                        bf16x2_to_f2(u1.x), bf16x2_to_f2(u1.y), bf16x2_to_f2(u1.z), bf16x2_to_f2(u1.w)};
#pragma unroll
                for (int hh = 0; hh < HPW; ++hh)
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        s01[hh] = f2_fma(c2[e], f2_pack(cur[hh][2 * e], cur[hh][2 * e + 1]), s01[hh]);
                        s23[hh] = f2_fma(c2[e + 1], f2_pack(cur[hh][2 * e + 2], cur[hh][2 * e + 3]), s23[hh]);
                    }
                if (a16 + 1 < C::RK / 16) {
#pragma unroll
                    for (int hh = 0; hh < HPW; ++hh) tmem_wait_ld_regs16(nxt[hh]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(tm_empty + buf);
                mbar_arrive(k_empty + kslot);
            }

            // ---- online softmax in base 2; p is rounded to bf16 for the V GEMM and l sums
            // the rounded values, so that numerator and denominator see the same weights
            float s2[HPW], mx[HPW];
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) {
                const float2 sp = f2_unpack(s01[hh]), sq = f2_unpack(s23[hh]);
                s2[hh] = row_ok ? ((sp.x + sp.y) + (sq.x + sq.y) + bias[hh]) * isc[hh] : -INFINITY;
                mx[hh] = s2[hh];
            }
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) mx[hh] = warp_max_f32(mx[hh]);
            const uint32_t pb = tile_n & 1;
            // P and alpha go to buffer tile_n & 1, last used by tile n - 2, whose V GEMM and
            // readers must be done with it
            if (tile_n >= 2) sync_ok(mbar_wait(d_empty + pb, ((tile_n >> 1) - 1) & 1, p.status, kFlagTimeout, 43));
#pragma unroll
            for (int hh = 0; hh < HPW; ++hh) {
                const float m_new = fmaxf(m[hh], mx[hh]);
                const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(m[hh] - m_new);
                const float pj = row_ok ? fast_exp2(s2[hh] - m_new) : 0.f;
                const __nv_bfloat16 pbf = __float2bfloat16_rn(pj);
                const uint16_t pbits = *reinterpret_cast<const uint16_t*>(&pbf);
                l[hh] = fmaf(l[hh], alpha, bf16_to_f32(pbits));
                m[hh] = m_new;
                *reinterpret_cast<uint16_t*>(p_s + pb * C::P_BYTES + p_off[hh]) = pbits;
                if (lane == 0) alpha_s[pb * (4 * C::HC) + qd * C::HC + hf0 + hh] = alpha;
            }
            if (g == 0 && nv < 32) {
                // rows past the context may hold any bits, and 0 * NaN is not 0: clear them in
                // the c^V slot before the V GEMM reads it
                const uint32_t vslot = (tile_n * 4 + qd) % C::NV;
                bool w = true;
                if (lane == 0) {
                    w = ok && mbar_wait(vt_full + (tile_n & 3), (tile_n >> 2) & 1, p.status, kFlagTimeout, 45);
                }
                ok = __shfl_sync(0xffffffffu, w, 0) && ok;
                __syncwarp();
                if (lane >= nv) {
                    uint8_t* row = v_s + size_t(vslot) * C::V_SLOT + lane * 128;
#pragma unroll
                    for (int pn = 0; pn < C::V_PANELS; ++pn)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4*>(row + pn * C::PANEL + c * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + pb);

            // ---- the previous tile's V GEMM, complete by now or shortly
            if (pending) accumulate(tile_n - 1);
            pending = true;
        }
        if (pending && ok) accumulate(tile_n - 1);
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
