// attention_pp.cuh -- the latent attention of "VideoMLA: Low-Rank Latent KV Cache
// for Minute-Scale Autoregressive Video Diffusion" (arXiv 2605.30351; absorbed
// form, App. E Eq. 8-10; scores Sec. 3.3 Eq. 7) for narrow latents, with two
// softmax warpgroups that take alternate key tiles.
//
// With d_c = 96 a key carries half the MMA work of d_c = 192 and the same
// exponentials per query row.  In the single-group kernel the two softmax warps
// of an SM sub-partition work on the same key tile in lockstep, so the MUFU
// idles while both load S, reduce the row max and store P.  Here group A (warps
// 2-5) owns the even key tiles and group B (warps 6-9) the odd ones, each with
// its own S buffer, P buffer, O accumulator and running (max, sum); a group's
// warp holds one query row per thread.  The groups share no buffer, so one
// group's exponentials overlap the other's tensor-memory traffic and waits.  At
// the end the two partial softmaxes merge exactly (each rescaled to the common
// max), then O / l goes through the W_uv,h epilogue as in the single-group
// kernel.  Key tiles are 96 keys, which fits O_A, O_B, S_A, S_B, P_A and P_B in
// tensor memory (Q lives in shared memory).
//
// Roles (352 threads):
//   warp 0     TMA producer: q_nope / W_uk (prologue), key tiles (latent blocks
//              + rotated RoPE keys) into an NS-stage ring, W_uv,h into the Q
//              region once the last score MMA has read Q
//   warp 1     tensor-memory owner; q_abs MMA, S_j = Q K_j^T into S_{j mod 2},
//              the W_uv epilogue MMA
//   warps 2-9  softmax groups A and B; q_abs -> bf16 Q and RoPE3D(q^R) -> fp16
//              into shared memory (prologue); merge and O / l (epilogue)
//   warp 10    O_{j mod 2} += P_{j mod 2} C_j
#pragma once

#include "attention.cuh"

namespace vmla {

// O_A, O_B (d_c each), S_A, S_B (96 each) and P_A, P_B (48 each) in 512 columns.
__host__ __device__ constexpr bool pingpong_fits(int dc) { return 2 * dc + 2 * 96 + 2 * 48 <= 512; }

template <int DC_, int DR_, int DN_, int DV_>
struct AttnPPCfg {
    static constexpr int DC = DC_, DR = DR_, DN = DN_, DV = DV_;
    static constexpr int W = DC + DR;
    static constexpr int BM = 128, BK = 96;
    static constexpr int C_ATOMS = (DC + 63) / 64;  // 64-column blocks (the last may be half used)
    static constexpr int C_ATOM = BK * 128;
    static constexpr int R_ROWB = DR * 2;           // bytes of rotated k^R per key (fp16)
    static constexpr uint32_t R_SW = DR == 16 ? SW32 : DR == 32 ? SW64 : SW128;
    static constexpr int STAGE = C_ATOMS * C_ATOM + BK * R_ROWB;
    static constexpr int QN_CHUNKS = DN / 16;
    static constexpr int QN_BYTES = QN_CHUNKS * BM * 32;
    static constexpr int WUK_ATOM = DN * 128, WUK_BYTES = C_ATOMS * WUK_ATOM;
    static constexpr int WUV_ATOM = DV * 128, WUV_BYTES = C_ATOMS * WUV_ATOM;
    static constexpr int OLAT_ATOM = BM * 128, OLAT_BYTES = C_ATOMS * OLAT_ATOM;
    // Q region: bf16 q_abs in 64-column K-major SW128 blocks, then fp16 rotated q^R;
    // after the key loop it takes W_uv,h
    static constexpr int Q_ATOM = BM * 128;
    static constexpr int QR_OFF = C_ATOMS * Q_ATOM;
    static constexpr int QBYTES = QR_OFF + BM * R_ROWB;
    static constexpr int TAIL = 1024 + 4096;  // alignment slack + barriers and the (max, sum) exchange
    static constexpr int NS = (6 * STAGE + QBYTES + TAIL <= 232448) ? 6 : (5 * STAGE + QBYTES + TAIL <= 232448) ? 5 : 4;
    static constexpr int OA = 0, OB = DC, SA = 2 * DC, SB = 2 * DC + BK, PA = 2 * DC + 2 * BK, PB = PA + BK / 2;
    static constexpr int OUT_COL = SA;  // the epilogue's output over S_A / S_B
    static constexpr int SMEM = NS * STAGE + QBYTES + TAIL;
    static constexpr int GROUP_WARPS = 4;
    static constexpr int THREADS = 32 * (3 + 2 * GROUP_WARPS);
    static_assert(pingpong_fits(DC) && DC % 32 == 0 && DC <= 256, "latent width");
    static_assert(DR == 16 || DR == 32 || DR == 64, "rope width");
    static_assert(DN % 16 == 0 && DV % 32 == 0 && OUT_COL + DV <= 512, "head widths");
    static_assert(QN_BYTES <= STAGE && WUK_BYTES <= STAGE && WUV_BYTES <= QBYTES && 2 * OLAT_BYTES <= NS * STAGE,
                  "prologue / epilogue buffers reuse pipeline stages and the Q region");
    static_assert(STAGE % 1024 == 0 && NS >= 4 && SMEM <= 232448, "shared memory budget");
};

struct AttnPPBarriers {
    uint64_t full[6], empty[6];
    uint64_t q_full, qabs_done, q_ready, s_all, wuv_full, pv_all, ml_ready, olat_ready, out_full, drain, drain2;
    uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
    uint32_t tmem_base;
    AbortState ab;
    float2 ml[2][128];  // per group and row: running max (raw score), running sum
};

template <class C>
__global__ void __launch_bounds__(352, 1) attention_pp_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
    constexpr int DC = C::DC, DR = C::DR, DN = C::DN, DV = C::DV, BM = C::BM, BK = C::BK, NS = C::NS;
    constexpr int NQ = BK / 32;  // 32-column chunks of a score row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* qreg = smem + NS * C::STAGE;
    AttnPPBarriers* bar = reinterpret_cast<AttnPPBarriers*>(qreg + C::QBYTES);
    AbortState* ab = &bar->ab;
    auto stage = [&](int s) { return smem + s * C::STAGE; };
    uint8_t* olat_hi = smem;                 // epilogue: O / l in bf16 hi and lo parts over the
    uint8_t* olat_lo = smem + C::OLAT_BYTES;  // first stages, idle once every PV MMA has completed
    griddep_launch_dependents();  // every CTA of this grid is resident or done before a dependent starts

    const int warp = warp_id(), lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * BM;
    const int nt = p.n_kt;  // key tiles of the window (>= 1); group g takes tiles g, g + 2, ...
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bar->full[s], 1);
            mbar_init(&bar->empty[s], 1);
        }
        mbar_init(&bar->q_full, 1);
        mbar_init(&bar->qabs_done, 1);
        mbar_init(&bar->q_ready, 2 * C::GROUP_WARPS);
        mbar_init(&bar->s_all, 1);
        mbar_init(&bar->wuv_full, 1);
        mbar_init(&bar->pv_all, 1);
        mbar_init(&bar->ml_ready, 2 * C::GROUP_WARPS);
        mbar_init(&bar->olat_ready, 2 * C::GROUP_WARPS);
        mbar_init(&bar->out_full, 1);
        mbar_init(&bar->drain, 1);
        mbar_init(&bar->drain2, 1);
        for (int g = 0; g < 2; ++g) {
            mbar_init(&bar->s_full[g], 1);
            mbar_init(&bar->s_free[g], C::GROUP_WARPS);
            mbar_init(&bar->p_full[g], C::GROUP_WARPS);
            mbar_init(&bar->pv_done[g], 1);
        }
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int r = 0; r < 3; ++r) {
                tma_prefetch_desc(&maps.cc[r]);
                tma_prefetch_desc(&maps.kr[r]);
            }
            tma_prefetch_desc(&maps.qn);
            tma_prefetch_desc(&maps.wuk);
            tma_prefetch_desc(&maps.wuv);
            mbar_arrive_expect_tx(&bar->q_full, C::QN_BYTES + C::WUK_BYTES);
            for (int c = 0; c < C::QN_CHUNKS; ++c)
                tma_load_4d(stage(NS - 2) + c * BM * 32, &maps.qn, &bar->q_full, c * 16, h, q0, b);
            for (int a = 0; a < C::C_ATOMS; ++a)
                tma_load_2d(stage(NS - 1) + a * C::WUK_ATOM, &maps.wuk, &bar->q_full, a * 64, h * DN);
            griddep_wait();  // the window is read only after the RoPE pre-pass has finished
            int issued = 0;
            bool qabs_seen = false, ok = true, wuv = false;
            for (int j = 0; j < nt; ++j) {
                const int s = j % NS;
                if (j >= NS) {
                    ok = mbar_wait(&bar->empty[s], ((j / NS) - 1) & 1, ab, to, 50);
                } else if (s >= NS - 2 && !qabs_seen) {  // stage still holds q_nope / W_uk
                    ok = qabs_seen = mbar_wait(&bar->qabs_done, 0, ab, to, 51);
                }
                if (!ok) break;
                int run, row, valid;
                key_tile<BK>(p, j, run, row, valid);
                mbar_arrive_expect_tx(&bar->full[s], C::STAGE);
                for (int a = 0; a < C::C_ATOMS; ++a)
                    tma_load_3d(stage(s) + a * C::C_ATOM, &maps.cc[run], &bar->full[s], a * 64, row, b);
                tma_load_3d(stage(s) + C::C_ATOMS * C::C_ATOM, &maps.kr[run], &bar->full[s], 0, row, b);
                issued = j + 1;
            }
            // W_uv,h for the epilogue into the Q region once the last score MMA has read Q
            if (ok && mbar_wait(&bar->s_all, 0, ab, to, 52)) {
                mbar_arrive_expect_tx(&bar->wuv_full, C::WUV_BYTES);
                for (int a = 0; a < C::C_ATOMS; ++a)
                    tma_load_2d(qreg + a * C::WUV_ATOM, &maps.wuv, &bar->wuv_full, a * 64, h * DV);
                wuv = true;
            }
            if (ab->flag) {  // let this CTA's copies land before it exits
                mbar_wait_drain(&bar->q_full, 0, to);
                if (wuv) mbar_wait_drain(&bar->wuv_full, 0, to);
                for (int j = issued > NS ? issued - NS : 0; j < issued; ++j)
                    mbar_wait_drain(&bar->full[j % NS], (j / NS) & 1, to);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ S issuer
        if (lane == 0) {
            bool ok = mbar_wait(&bar->q_full, 0, ab, to, 60);
            if (ok) {
                tc_fence_after();
                // q_abs [128 x DC] = q_nope [128 x DN] . W_uk,h [DN x DC] into O_A's columns
                constexpr uint32_t id_qabs = idesc_bf16_f32(128, DC, false, true);
                const uint32_t sq = smem_u32(stage(NS - 2)), sw = smem_u32(stage(NS - 1));
#pragma unroll
                for (int k = 0; k < C::QN_CHUNKS; ++k)
                    umma_ss(tmem + C::OA, sdesc(sq + k * BM * 32, 16, 256, SW32),
                            sdesc(sw + k * 2048, C::WUK_ATOM, 1024, SW128), id_qabs, k > 0);
                umma_commit(&bar->qabs_done);
                ok = mbar_wait(&bar->q_ready, 0, ab, to, 61);
            }
            constexpr uint32_t id_s = idesc_bf16_f32(128, BK, false, false);
            constexpr uint32_t id_s_rope = idesc_f16_f32(128, BK, false, false);
            const uint32_t sq = smem_u32(qreg);
            for (int j = 0; ok && j < nt; ++j) {
                // S_j = Q . K_j^T : K = DC latent (bf16) + DR rotated rope (fp16) columns
                const int g = j & 1, k = j >> 1, s = j % NS;
                ok = mbar_wait(&bar->full[s], (j / NS) & 1, ab, to, 62);
                if (ok && j >= 2) ok = mbar_wait(&bar->s_free[g], (k - 1) & 1, ab, to, 63);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(stage(s));
                const uint32_t sd = tmem + (g ? C::SB : C::SA);
#pragma unroll
                for (int kk = 0; kk < DC / 16; ++kk)
                    umma_ss(sd, sdesc(sq + (kk / 4) * C::Q_ATOM + (kk % 4) * 32, 16, 1024, SW128),
                            sdesc(st + (kk / 4) * C::C_ATOM + (kk % 4) * 32, 16, 1024, SW128), id_s, kk > 0);
#pragma unroll
                for (int kk = 0; kk < DR / 16; ++kk)
                    umma_ss(sd, sdesc(sq + C::QR_OFF + kk * 32, 16, 8 * C::R_ROWB, C::R_SW),
                            sdesc(st + C::C_ATOMS * C::C_ATOM + kk * 32, 16, 8 * C::R_ROWB, C::R_SW), id_s_rope, 1);
                umma_commit(&bar->s_full[g]);
            }
            if (ok) {
                umma_commit(&bar->s_all);  // Q is no longer read: the producer may put W_uv there
                // out [128 x DV] = O_lat [128 x DC] . W_uv,h^T: O_lat as bf16 hi and lo parts
                ok = mbar_wait(&bar->wuv_full, 0, ab, to, 64) && mbar_wait(&bar->olat_ready, 0, ab, to, 65);
                if (ok) {
                    tc_fence_after();
                    constexpr uint32_t id_o = idesc_bf16_f32(128, DV, false, false);
                    const uint32_t bw = smem_u32(qreg), ao = smem_u32(olat_hi), ao2 = smem_u32(olat_lo);
#pragma unroll
                    for (int k = 0; k < DC / 16; ++k) {
                        const int a = k / 4;
                        const uint64_t bd = sdesc(bw + a * C::WUV_ATOM + (k % 4) * 32, 16, 1024, SW128);
                        const uint32_t off = a * C::OLAT_ATOM + (k % 4) * 32;
                        umma_ss(tmem + C::OUT_COL, sdesc(ao + off, 16, 1024, SW128), bd, id_o, k > 0);
                        umma_ss(tmem + C::OUT_COL, sdesc(ao2 + off, 16, 1024, SW128), bd, id_o, 1);
                    }
                    umma_commit(&bar->out_full);
                }
            }
            if (!ok) {  // no MMA may still run when the tensor memory is released
                umma_commit(&bar->drain);
                mbar_wait_drain(&bar->drain, 0, to);
            }
        }
    } else if (warp == 2 + 2 * C::GROUP_WARPS) {
        // ------------------------------------------------------------ PV issuer
        if (lane == 0) {
            constexpr uint32_t id_pv = idesc_bf16_f32(128, DC, false, true);
            bool ok = true;
            for (int j = 0; ok && j < nt; ++j) {
                const int g = j & 1, k = j >> 1;
                ok = mbar_wait(&bar->p_full[g], k & 1, ab, to, 66);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(stage(j % NS));
                const uint32_t od = tmem + (g ? C::OB : C::OA), pa = tmem + (g ? C::PB : C::PA);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    umma_ts(od, pa + kk * 8, sdesc(st + kk * 2048, C::C_ATOM, 1024, SW128), id_pv, j >= 2 || kk > 0);
                umma_commit(&bar->empty[j % NS]);
                umma_commit(&bar->pv_done[g]);
            }
            if (ok) umma_commit(&bar->pv_all);
            umma_commit(&bar->drain2);
            mbar_wait_drain(&bar->drain2, 0, to);
        }
    } else {
        // ------------------------------------------------------------ softmax groups
        // warps 2-5 (group A) and 6-9 (group B); a warp may only touch TMEM lanes
        // 32 (warp % 4) .. + 31, so thread `lane` of either group's warp owns query
        // row r = 32 (warp % 4) + lane of the tile.
        const int q4 = warp & 3;
        const int g = (warp - 2) / C::GROUP_WARPS;
        const int r = q4 * 32 + lane;
        const uint32_t tq = tmem + (uint32_t(q4 * 32) << 16);
        const float sl = p.scale_log2;
        const int cnt_g = (nt - g + 1) >> 1, cnt_o = (nt - (1 - g) + 1) >> 1;  // tiles of this / the other group

        // prologue: Q = [bf16(q_abs) | fp16(RoPE3D(q^R))] into the swizzled K-major Q
        // region; the groups take alternate 32-column chunks of q_abs
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bar->qabs_done, 0, ab, to, 70) && !ab->flag);
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 32 * g; c < DC; c += 64) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tq + C::OA + c, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                uint8_t* row_base = qreg + (c / 64) * C::Q_ATOM + r * 128;
                const int kc0 = (c % 64) / 8;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    *reinterpret_cast<uint4*>(row_base + (((kc0 + i) ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
            if (g == 0) {
                const int i = q0 + r;
                uint32_t qr[DR / 2];
#pragma unroll
                for (int e = 0; e < DR / 2; ++e) qr[e] = 0u;
                if (i < p.Nq) {
                    const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + ((size_t(b) * p.Nq + i) * p.H + h) * DR);
                    const int L = p.q_first + i;
                    const int tq_ = L / p.T_f;
                    const int pq = L - tq_ * p.T_f;
                    const int hq = pq / p.grid_w, wq = pq - (pq / p.grid_w) * p.grid_w;
#pragma unroll
                    for (int c = 0; c < DR / 8; ++c) {
                        const uint4 v = __ldg(src + c);
                        qr[4 * c + 0] = rotate_pair(v.x, rope_theta(p, 4 * c + 0, tq_, hq, wq));
                        qr[4 * c + 1] = rotate_pair(v.y, rope_theta(p, 4 * c + 1, tq_, hq, wq));
                        qr[4 * c + 2] = rotate_pair(v.z, rope_theta(p, 4 * c + 2, tq_, hq, wq));
                        qr[4 * c + 3] = rotate_pair(v.w, rope_theta(p, 4 * c + 3, tq_, hq, wq));
                    }
                }
                // rows of R_ROWB bytes, 16-byte chunk index XOR-ed by address bits
                // [7, 7 + log2(R_ROWB / 16)): the 32B / 64B / 128B swizzles
                uint8_t* row_base = qreg + C::QR_OFF + r * C::R_ROWB;
                constexpr int NCH16 = C::R_ROWB / 16;
#pragma unroll
                for (int e = 0; e < NCH16; ++e) {
                    const int sw = ((r * C::R_ROWB) >> 7) & (NCH16 - 1);
                    *reinterpret_cast<uint4*>(row_base + ((e ^ sw) << 4)) =
                        make_uint4(qr[4 * e], qr[4 * e + 1], qr[4 * e + 2], qr[4 * e + 3]);
                }
            }
            fence_proxy_async_smem();  // generic stores -> MMA operand reads
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->q_ready);
        }

        griddep_wait();  // the stores below may not overtake the RoPE pre-pass

        // main loop over this group's tiles j = g, g + 2, ...; one row per thread,
        // register c of chunk q = score column 32 q + c
        const uint32_t s_col = g ? C::SB : C::SA, p_col = g ? C::PB : C::PA, o_col = g ? C::OB : C::OA;
        float m_used = -INFINITY, l_run = 0.f;
        for (int j = g; ok && j < nt; j += 2) {
            const int k = j >> 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->s_full[g], k & 1, ab, to, 71));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[NQ][32];
#pragma unroll
            for (int q = 0; q < NQ; ++q) tmem_ld_32x32b_x32(tq + s_col + 32 * q, sv[q]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->s_free[g]);

            int run, row, valid;
            key_tile<BK>(p, j, run, row, valid);
            if (valid < BK) {  // ragged last tile of a run: mask the missing keys
#pragma unroll
                for (int q = 0; q < NQ; ++q)
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (32 * q + c >= valid) sv[q][c] = 0xff800000u;  // -inf
            }
            float mxq[NQ];  // two independent max chains per 32-column chunk
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                float m0 = __uint_as_float(sv[q][0]), m1 = __uint_as_float(sv[q][16]);
#pragma unroll
                for (int c = 1; c < 15; c += 2) {
                    m0 = fmax3(m0, __uint_as_float(sv[q][c]), __uint_as_float(sv[q][c + 1]));
                    m1 = fmax3(m1, __uint_as_float(sv[q][16 + c]), __uint_as_float(sv[q][16 + c + 1]));
                }
                mxq[q] = fmaxf(fmax3(m0, m1, __uint_as_float(sv[q][15])), __uint_as_float(sv[q][31]));
            }
            float mx = mxq[0];
#pragma unroll
            for (int q = 1; q < NQ; ++q) mx = fmaxf(mx, mxq[q]);
            // Move the max only when some row's max grew by more than 2^8 in probability
            // units; otherwise keep the stale max (exact, p <= 256 fits bf16 / fp32).
            float f_resc = 1.f;
            bool rescale = false;
            if (k == 0) {
                m_used = mx;
            } else if (__any_sync(0xffffffffu, (mx - m_used) * sl > 8.0f)) {
                const float mn = fmaxf(m_used, mx);
                f_resc = ex2((m_used - mn) * sl);
                m_used = mn;
                l_run *= f_resc;
                rescale = true;
            }
            // P = exp2(s sl - m sl) as bf16 pairs: column c of P_g holds keys 2c, 2c + 1
            const float2 sl2 = make_float2(sl, sl);
            const float2 nm = make_float2(-m_used * sl, -m_used * sl);
            float2 acc[NQ];  // one row-sum chain per chunk
            uint32_t pk[NQ][16];
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                acc[q] = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float2 x = __ffma2_rn(
                        make_float2(__uint_as_float(sv[q][2 * c]), __uint_as_float(sv[q][2 * c + 1])), sl2, nm);
                    const float2 e = make_float2(ex2(x.x), ex2(x.y));
                    acc[q] = __fadd2_rn(acc[q], e);
                    pk[q][c] = pack_bf16(e.x, e.y);
                }
            }
#pragma unroll
            for (int q = 0; q < NQ; ++q) l_run += acc[q].x + acc[q].y;
            // P_g and O_g are free once this group's previous PV has completed
            if (k >= 1) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done[g], (k - 1) & 1, ab, to, 72));
                if (!ok) break;
                tc_fence_after();
            }
#pragma unroll
            for (int q = 0; q < NQ; ++q) tmem_st_32x32b_x16(tq + p_col + 16 * q, pk[q]);
            if (rescale) {  // O_g *= f
#pragma unroll 1
                for (int cc = 0; cc < DC; cc += 32) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tq + o_col + cc, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f_resc);
                    tmem_st_32x32b_x32(tq + o_col + cc, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->p_full[g]);
        }

        // merge the two groups' partial softmaxes to the common max
        if (ok) {
            bar->ml[g][r] = make_float2(cnt_g ? m_used : -INFINITY, cnt_g ? l_run : 0.f);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->ml_ready);
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->ml_ready, 0, ab, to, 74) && !ab->flag);
        }
        float f_a = 0.f, f_b = 0.f, inv = 0.f, m_fin = 0.f, l_fin = 0.f;
        if (ok) {
            const float2 own = bar->ml[g][r], oth = bar->ml[1 - g][r];
            m_fin = fmaxf(own.x, oth.x);
            const float f_own = cnt_g ? ex2((own.x - m_fin) * sl) : 0.f;
            const float f_oth = cnt_o ? ex2((oth.x - m_fin) * sl) : 0.f;
            l_fin = own.y * f_own + oth.y * f_oth;
            inv = 1.0f / l_fin;
            f_a = g ? f_oth : f_own;
            f_b = g ? f_own : f_oth;
            // both accumulators final: every PV MMA has completed
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_all, 0, ab, to, 75) && !ab->flag);
        }
        if (ok) {
            tc_fence_after();
            // O_lat = (f_A O_A + f_B O_B) / l as bf16 hi + lo parts, K-major SW128; the
            // groups take alternate 32-column chunks
            const bool use_b = nt > 1;
#pragma unroll 1
            for (int c = 32 * g; c < DC; c += 64) {
                uint32_t oa[32], ob[32];
                tmem_ld_32x32b_x32(tq + C::OA + c, oa);
                if (use_b) tmem_ld_32x32b_x32(tq + C::OB + c, ob);
                tmem_wait_ld();
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float v0 = __uint_as_float(oa[2 * e]) * f_a, v1 = __uint_as_float(oa[2 * e + 1]) * f_a;
                    if (use_b) {
                        v0 = fmaf(__uint_as_float(ob[2 * e]), f_b, v0);
                        v1 = fmaf(__uint_as_float(ob[2 * e + 1]), f_b, v1);
                    }
                    split_bf16(v0 * inv, v1 * inv, hi[e], lo[e]);
                }
                const int base = (c / 64) * C::OLAT_ATOM + r * 128;
                const int kc0 = (c % 64) / 8;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int off = base + (((kc0 + i) ^ (r & 7)) << 4);
                    *reinterpret_cast<uint4*>(olat_hi + off) =
                        make_uint4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
                    *reinterpret_cast<uint4*>(olat_lo + off) =
                        make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->olat_ready);

            const int i = q0 + r;
            if (p.lse != nullptr && g == 0 && i < p.Nq)
                p.lse[(size_t(b) * p.Nq + i) * p.H + h] = (m_fin * sl + __log2f(l_fin)) * 0.69314718055994531f;

            // out rows, one per thread; the groups take alternate 32-column chunks
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->out_full, 0, ab, to, 77) && !ab->flag);
            if (ok) {
                tc_fence_after();
                __nv_bfloat16* dst = p.out + ((size_t(b) * p.Nq + i) * p.H + h) * DV;
#pragma unroll 1
                for (int c = 32 * g; c < DV; c += 64) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tq + C::OUT_COL + c, v);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                    if (i < p.Nq) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
                        for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace vmla
