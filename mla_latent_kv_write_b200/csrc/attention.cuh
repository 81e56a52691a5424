// attention.cuh -- latent multi-head attention of "VideoMLA: Low-Rank Latent KV
// Cache for Minute-Scale Autoregressive Video Diffusion" (arXiv 2605.30351) in
// the absorbed inference form of App. E:
//   q_abs  = W_uk,h^T q^nope                            (Eq. 8-9)
//   s_ij   = (q_abs . c_j + RoPE3D(q^R_i) . RoPE3D(k^R_j)) / sqrt(d_nope + d_rope)
//                                                        (Eq. 7, Eq. 12)
//   o_i,h  = W_uv,h ( sum_j softmax_j(s_ij) c_j )        (Eq. 10 without W_O)
// over every key of the ring window (App. D.4), with keys and queries rotated
// by their window-local (t, h, w) positions (App. D.5).
//
// One CTA per (128-query tile, head, batch element); 256 threads:
//   warp 0     TMA producer: q_nope / W_uk (prologue), key tiles (128 keys x
//              [c | k^R]) into a 3-stage ring, W_uv (epilogue)
//   warp 1     tcgen05.mma issuer and tensor-memory owner
//   warps 2-3  RoPE transform: rotate each landed k^R tile in shared memory
//   warps 4-7  softmax: q_abs -> bf16 Q in TMEM, q^R rotation, fp32 online
//              softmax (row max / sum reduced across the 4 threads of a row
//              with warp shuffles), P -> TMEM, O rescale, normalisation,
//              W_uv epilogue and the output stores
// Tensor memory (512 columns, fp32 unless noted):
//   O [0, d_c)  S [d_c, d_c+128)  P (bf16 pairs) [+128, +64)
//   Q (bf16 pairs of q_abs, then fp16 pairs of the rotated q^R)
// Both contractions read their A operand from TMEM (Q for S = Q K^T, P for
// O += P C) and their B operand from the swizzled shared-memory key tile: the
// content part is K-major for S and MN-major for P C, so one copy serves both.
#pragma once

#include "ptx.cuh"

namespace vmla {

constexpr int kAttnTableMax = 2048;  // float2 (cos, sin) entries of the rope tables

struct AttnParams {
    int Nq, H;
    int T_f, grid_w, slots, oldest;
    int seg_start[2], seg_len[2];  // valid physical key rows: up to two contiguous runs
    int n_kt;                      // key tiles
    int q_first;                   // logical window index of query 0
    int n_t, n_h, n_w;             // rope pairs per axis
    int tab_h_off, tab_w_off, tab_total;
    float omega[32];               // rope frequency of each pair
    float scale_log2;              // log2(e) / sqrt(d_nope + d_rope)
    const __nv_bfloat16* q_rope;   // [B, Nq, H, DR]
    __nv_bfloat16* out;            // [B, Nq, H, DV]
    float* lse;                    // [B, Nq, H] or null
    uint64_t timeout_ns;
};

template <int DC_, int DR_, int DN_, int DV_>
struct AttnCfg {
    static constexpr int DC = DC_, DR = DR_, DN = DN_, DV = DV_;
    static constexpr int W = DC + DR;  // cached scalars per token
    static constexpr int BM = 128, BK = 128, NS = 3;
    static constexpr int C_ATOMS = DC / 64;
    static constexpr int C_ATOM = BK * 128;           // one 64-column block of the key tile
    static constexpr int R_ROWB = DR * 2;             // bytes of k^R per key
    static constexpr uint32_t R_SW = DR == 16 ? SW32 : DR == 32 ? SW64 : SW128;
    static constexpr int STAGE = C_ATOMS * C_ATOM + BK * R_ROWB;
    static constexpr int O_COL = 0, S_COL = DC, P_COL = DC + BK, Q_COL = DC + BK + BK / 2;
    static constexpr int TMEM_END = Q_COL + W / 2;
    static constexpr int QN_CHUNKS = DN / 16;
    static constexpr int QN_BYTES = QN_CHUNKS * BM * 32;
    static constexpr int WUK_ATOM = DN * 128, WUK_BYTES = C_ATOMS * WUK_ATOM;
    static constexpr int WUV_ATOM = DV * 128, WUV_BYTES = C_ATOMS * WUV_ATOM;
    static constexpr int OLAT_ATOM = BM * 128;
    static constexpr int SMEM = NS * STAGE + kAttnTableMax * 8 + 512 + 1024;
    static constexpr int THREADS = 256;
    static_assert(DC % 64 == 0 && DC <= 256, "latent width");
    static_assert(DR == 16 || DR == 32 || DR == 64, "rope width");
    static_assert(DN % 16 == 0 && DV % 32 == 0 && DV <= 256, "head widths");
    static_assert(TMEM_END <= 512, "tensor memory budget");
    static_assert(QN_BYTES <= STAGE && WUK_BYTES <= STAGE && WUV_BYTES <= STAGE &&
                  C_ATOMS * OLAT_ATOM <= STAGE, "prologue / epilogue buffers reuse pipeline stages");
};

struct AttnBarriers {
    uint64_t full[4], empty[4], rot[4];
    uint64_t q_full, qabs_done, q_ready, s_full, s_free, p_full, pv_done, olat_ready, out_full, drain;
    uint32_t tmem_base;
    AbortState ab;
};

template <int BK>
__device__ __forceinline__ void key_tile(const AttnParams& p, int j, int& start, int& valid) {
    const int t0 = (p.seg_len[0] + BK - 1) / BK;
    const int s = j < t0 ? 0 : 1;
    const int jj = j < t0 ? j : j - t0;
    start = p.seg_start[s] + jj * BK;
    valid = min(BK, p.seg_len[s] - jj * BK);
}

// (cos, sin) of pair ``pr`` at grid position (t, hh, ww).
__device__ __forceinline__ float2 rope_cs(const float2* tab, const AttnParams& p, int pr, int t, int hh, int ww) {
    if (pr < p.n_t) return tab[t * p.n_t + pr];
    if (pr < p.n_t + p.n_h) return tab[p.tab_h_off + hh * p.n_h + (pr - p.n_t)];
    return tab[p.tab_w_off + ww * p.n_w + (pr - p.n_t - p.n_h)];
}

// Rotate one packed bf16 pair (x in the low half) by (cos, sin); the rotated
// pair is packed as fp16: the RoPE part of the score contraction runs as its own
// fp16 x fp16 MMAs, whose 11-bit significand keeps the rounding of the rotated
// vectors 8x below bf16 (values are O(10), far inside the fp16 range).
__device__ __forceinline__ uint32_t rotate_pair(uint32_t v, float2 cs) {
    const float x = bf16_lo(v), y = bf16_hi(v);
    return pack_f16(x * cs.x - y * cs.y, x * cs.y + y * cs.x);
}

template <class C>
__global__ void __launch_bounds__(256, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tm_cc, const __grid_constant__ CUtensorMap tm_cr,
                     const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_wuk,
                     const __grid_constant__ CUtensorMap tm_wuv, const AttnParams p) {
    constexpr int DC = C::DC, DR = C::DR, DN = C::DN, DV = C::DV, BM = C::BM, BK = C::BK, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float2* tab = reinterpret_cast<float2*>(smem + NS * C::STAGE);
    AttnBarriers* bar = reinterpret_cast<AttnBarriers*>(smem + NS * C::STAGE + kAttnTableMax * 8);
    AbortState* ab = &bar->ab;
    auto stage = [&](int s) { return smem + s * C::STAGE; };

    const int warp = warp_id(), lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * BM;
    const int nt = p.n_kt;
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bar->full[s], 1);
            mbar_init(&bar->empty[s], 1);
            mbar_init(&bar->rot[s], 2);
        }
        mbar_init(&bar->q_full, 1);
        mbar_init(&bar->qabs_done, 1);
        mbar_init(&bar->q_ready, 4);
        mbar_init(&bar->s_full, 1);
        mbar_init(&bar->s_free, 4);
        mbar_init(&bar->p_full, 4);
        mbar_init(&bar->pv_done, 1);
        mbar_init(&bar->olat_ready, 4);
        mbar_init(&bar->out_full, 1);
        mbar_init(&bar->drain, 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bar->tmem_base, 512);
        tmem_relinquish();
    }
    // rope tables: [t][n_t] then [h][n_h] then [w][n_w] of (cos, sin)(pos * omega)
    for (int e = threadIdx.x; e < p.tab_total; e += blockDim.x) {
        int pos, pr;
        if (e < p.tab_h_off) {
            pos = e / p.n_t;
            pr = e - pos * p.n_t;
        } else if (e < p.tab_w_off) {
            const int e2 = e - p.tab_h_off;
            pos = e2 / p.n_h;
            pr = p.n_t + (e2 - pos * p.n_h);
        } else {
            const int e2 = e - p.tab_w_off;
            pos = e2 / p.n_w;
            pr = p.n_t + p.n_h + (e2 - pos * p.n_w);
        }
        float sn, cs;
        sincosf(float(pos) * p.omega[pr], &sn, &cs);
        tab[e] = make_float2(cs, sn);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_cc);
            tma_prefetch_desc(&tm_cr);
            tma_prefetch_desc(&tm_qn);
            tma_prefetch_desc(&tm_wuk);
            tma_prefetch_desc(&tm_wuv);
            mbar_arrive_expect_tx(&bar->q_full, C::QN_BYTES + C::WUK_BYTES);
            for (int c = 0; c < C::QN_CHUNKS; ++c)
                tma_load_4d(stage(NS - 2) + c * BM * 32, &tm_qn, &bar->q_full, c * 16, h, q0, b);
            for (int a = 0; a < C::C_ATOMS; ++a)
                tma_load_2d(stage(NS - 1) + a * C::WUK_ATOM, &tm_wuk, &bar->q_full, a * 64, h * DN);
            int issued = 0;
            bool qabs_seen = false;
            for (int j = 0; j <= nt; ++j) {
                const int s = j % NS;
                bool ok = true;
                if (j >= NS) {
                    ok = mbar_wait(&bar->empty[s], ((j / NS) - 1) & 1, ab, to, 10);
                } else if (s >= NS - 2 && !qabs_seen) {  // stage still holds q_nope / W_uk
                    ok = qabs_seen = mbar_wait(&bar->qabs_done, 0, ab, to, 11);
                }
                if (!ok) break;
                if (j < nt) {
                    int start, valid;
                    key_tile<BK>(p, j, start, valid);
                    mbar_arrive_expect_tx(&bar->full[s], C::STAGE);
                    for (int a = 0; a < C::C_ATOMS; ++a)
                        tma_load_3d(stage(s) + a * C::C_ATOM, &tm_cc, &bar->full[s], a * 64, start, b);
                    tma_load_3d(stage(s) + C::C_ATOMS * C::C_ATOM, &tm_cr, &bar->full[s], DC, start, b);
                } else {
                    mbar_arrive_expect_tx(&bar->full[s], C::WUV_BYTES);
                    for (int a = 0; a < C::C_ATOMS; ++a)
                        tma_load_2d(stage(s) + a * C::WUV_ATOM, &tm_wuv, &bar->full[s], a * 64, h * DV);
                }
                issued = j + 1;
            }
            if (ab->flag) {  // let this CTA's copies land before it exits
                mbar_wait_drain(&bar->q_full, 0, to);
                for (int j = issued > NS ? issued - NS : 0; j < issued; ++j)
                    mbar_wait_drain(&bar->full[j % NS], (j / NS) & 1, to);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = mbar_wait(&bar->q_full, 0, ab, to, 30);
            if (ok) {
                tc_fence_after();
                // q_abs [128 x DC] = q_nope [128 x DN] . W_uk,h [DN x DC]   (A: K-major SW32 chunks,
                // B: MN-major SW128 blocks of 64 latent columns)
                constexpr uint32_t id_qabs = idesc_bf16_f32(128, DC, false, true);
                const uint32_t sq = smem_u32(stage(NS - 2)), sw = smem_u32(stage(NS - 1));
#pragma unroll
                for (int k = 0; k < C::QN_CHUNKS; ++k)
                    umma_ss(tmem + C::O_COL, sdesc(sq + k * BM * 32, 16, 256, SW32),
                            sdesc(sw + k * 2048, C::WUK_ATOM, 1024, SW128), id_qabs, k > 0);
                umma_commit(&bar->qabs_done);
                ok = mbar_wait(&bar->q_ready, 0, ab, to, 31);
            }
            constexpr uint32_t id_s = idesc_bf16_f32(128, BK, false, false);
            constexpr uint32_t id_s_rope = idesc_f16_f32(128, BK, false, false);
            constexpr uint32_t id_pv = idesc_bf16_f32(128, DC, false, true);
            for (int j = 0; ok && j <= nt; ++j) {
                if (j < nt) {
                    // S_j = Q . K_j^T : K = DC latent + DR rope columns, 16 per MMA
                    const int s = j % NS;
                    ok = mbar_wait(&bar->rot[s], (j / NS) & 1, ab, to, 32);
                    if (ok && j > 0) ok = mbar_wait(&bar->s_free, (j - 1) & 1, ab, to, 33);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t st = smem_u32(stage(s));
#pragma unroll
                    for (int k = 0; k < C::W / 16; ++k) {
                        if (k < DC / 16)  // latent part: bf16 x bf16
                            umma_ts(tmem + C::S_COL, tmem + C::Q_COL + k * 8,
                                    sdesc(st + (k / 4) * C::C_ATOM + (k % 4) * 32, 16, 1024, SW128), id_s, k > 0);
                        else              // rotated RoPE part: fp16 x fp16
                            umma_ts(tmem + C::S_COL, tmem + C::Q_COL + k * 8,
                                    sdesc(st + C::C_ATOMS * C::C_ATOM + (k - DC / 16) * 32, 16, 8 * C::R_ROWB, C::R_SW),
                                    id_s_rope, 1);
                    }
                    umma_commit(&bar->s_full);
                }
                if (j > 0) {
                    // O += P_{j-1} . C_{j-1} : B is the latent block of the same tile, MN-major
                    const int jj = j - 1, sp = jj % NS;
                    ok = mbar_wait(&bar->p_full, jj & 1, ab, to, 34);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t st = smem_u32(stage(sp));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_ts(tmem + C::O_COL, tmem + C::P_COL + k * 8, sdesc(st + k * 2048, C::C_ATOM, 1024, SW128),
                                id_pv, (jj > 0 || k > 0));
                    umma_commit(&bar->empty[sp]);
                    umma_commit(&bar->pv_done);
                }
            }
            if (ok) {
                // out [128 x DV] = (O_hi + O_lo) [128 x DC] . W_uv,h^T  (all K-major SW128):
                // O / l is split into two bf16 parts so that its rounding stays ~2^-16
                const int sw_ = nt % NS, so = (nt + 1) % NS, so2 = (nt + 2) % NS;
                ok = mbar_wait(&bar->full[sw_], (nt / NS) & 1, ab, to, 35) &&
                     mbar_wait(&bar->olat_ready, 0, ab, to, 36);
                if (ok) {
                    tc_fence_after();
                    constexpr uint32_t id_o = idesc_bf16_f32(128, DV, false, false);
                    const uint32_t ao = smem_u32(stage(so)), ao2 = smem_u32(stage(so2)), bw = smem_u32(stage(sw_));
#pragma unroll
                    for (int k = 0; k < DC / 16; ++k) {
                        const uint64_t bd = sdesc(bw + (k / 4) * C::WUV_ATOM + (k % 4) * 32, 16, 1024, SW128);
                        const uint32_t off = (k / 4) * C::OLAT_ATOM + (k % 4) * 32;
                        umma_ss(tmem + C::S_COL, sdesc(ao + off, 16, 1024, SW128), bd, id_o, k > 0);
                        umma_ss(tmem + C::S_COL, sdesc(ao2 + off, 16, 1024, SW128), bd, id_o, 1);
                    }
                    umma_commit(&bar->out_full);
                }
            }
            if (!ok) {  // no MMA may still run when the tensor memory is released
                umma_commit(&bar->drain);
                mbar_wait_drain(&bar->drain, 0, to);
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ RoPE transform
        const int tid = threadIdx.x - 64;
        constexpr int CHUNKS = C::R_ROWB / 16;
        for (int j = 0; j < nt; ++j) {
            const int s = j % NS;
            if (!__all_sync(0xffffffffu, mbar_wait(&bar->full[s], (j / NS) & 1, ab, to, 20))) break;
            int start, valid;
            key_tile<BK>(p, j, start, valid);
            uint8_t* kr = stage(s) + C::C_ATOMS * C::C_ATOM;
            for (int rr = tid; rr < BK; rr += 64) {
                if (rr < valid) {
                    const int R = start + rr;
                    const int slot = R / p.T_f;
                    const int pp = R - slot * p.T_f;
                    int t = slot - p.oldest;
                    if (t < 0) t += p.slots;
                    const int hh = pp / p.grid_w;
                    const int ww = pp - hh * p.grid_w;
                    uint8_t* row = kr + rr * C::R_ROWB;
                    const int sw = (rr * C::R_ROWB >> 7) & (CHUNKS - 1);
#pragma unroll
                    for (int c = 0; c < CHUNKS; ++c) {
                        uint4* ptr = reinterpret_cast<uint4*>(row + ((c ^ sw) << 4));
                        uint4 v = *ptr;
                        v.x = rotate_pair(v.x, rope_cs(tab, p, 4 * c + 0, t, hh, ww));
                        v.y = rotate_pair(v.y, rope_cs(tab, p, 4 * c + 1, t, hh, ww));
                        v.z = rotate_pair(v.z, rope_cs(tab, p, 4 * c + 2, t, hh, ww));
                        v.w = rotate_pair(v.w, rope_cs(tab, p, 4 * c + 3, t, hh, ww));
                        *ptr = v;
                    }
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->rot[s]);
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        const int w4 = warp - 4;
        const int quad = lane & 3;
        const uint32_t tl = tmem + (uint32_t(w4 * 32) << 16);  // this warp's TMEM lane quarter
        const uint32_t tl16 = tl + (16u << 16);
        const float sl = p.scale_log2;

        // prologue: Q = [bf16(q_abs) | fp16(RoPE3D(q^R))] into TMEM, one row per thread
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bar->qabs_done, 0, ab, to, 40) && !ab->flag);
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < DC; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tl + C::O_COL + c, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                tmem_st_32x32b_x16(tl + C::Q_COL + c / 2, pk);
            }
            const int r = w4 * 32 + lane;
            const int i = q0 + r;
            uint32_t qr[DR / 2];
#pragma unroll
            for (int e = 0; e < DR / 2; ++e) qr[e] = 0u;
            if (i < p.Nq) {
                const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + ((size_t(b) * p.Nq + i) * p.H + h) * DR);
                const int L = p.q_first + i;
                const int tq = L / p.T_f;
                const int pq = L - tq * p.T_f;
                const int hq = pq / p.grid_w, wq = pq - (pq / p.grid_w) * p.grid_w;
#pragma unroll
                for (int c = 0; c < DR / 8; ++c) {
                    const uint4 v = __ldg(src + c);
                    qr[4 * c + 0] = rotate_pair(v.x, rope_cs(tab, p, 4 * c + 0, tq, hq, wq));
                    qr[4 * c + 1] = rotate_pair(v.y, rope_cs(tab, p, 4 * c + 1, tq, hq, wq));
                    qr[4 * c + 2] = rotate_pair(v.z, rope_cs(tab, p, 4 * c + 2, tq, hq, wq));
                    qr[4 * c + 3] = rotate_pair(v.w, rope_cs(tab, p, 4 * c + 3, tq, hq, wq));
                }
            }
            if constexpr (DR == 16) {
                tmem_st_32x32b_x8(tl + C::Q_COL + DC / 2, qr);
            } else if constexpr (DR == 32) {
                tmem_st_32x32b_x16(tl + C::Q_COL + DC / 2, qr);
            } else {
                tmem_st_32x32b_x32(tl + C::Q_COL + DC / 2, qr);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->q_ready);
        }

        // main loop.  16x256b layout: this thread holds rows
        //   R0 = w4*32 + lane/4, R1 = R0 + 8 (lanes 0-15 of the quarter) and
        //   R2 = R0 + 16, R3 = R0 + 24 (lanes 16-31), 32 columns of each.
        float m_used[4], l_part[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            m_used[k] = 0.f;
            l_part[k] = 0.f;
        }
        for (int j = 0; ok && j < nt; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->s_full, j & 1, ab, to, 41));
            if (!ok) break;
            tc_fence_after();
            uint32_t sa[2][32], sb[2][32];
            tmem_ld_16x256b_x8(tl + C::S_COL, sa[0]);
            tmem_ld_16x256b_x8(tl + C::S_COL + 64, sa[1]);
            tmem_ld_16x256b_x8(tl16 + C::S_COL, sb[0]);
            tmem_ld_16x256b_x8(tl16 + C::S_COL + 64, sb[1]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->s_free);

            int start, valid;
            key_tile<BK>(p, j, start, valid);
            if (valid < BK) {  // ragged last tile of a segment: mask the missing keys
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int col = 64 * c + 8 * k + 2 * quad + e;
                            if (col >= valid) {
                                sa[c][4 * k + e] = sa[c][4 * k + 2 + e] = 0xff800000u;  // -inf
                                sb[c][4 * k + e] = sb[c][4 * k + 2 + e] = 0xff800000u;
                            }
                        }
            }
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    mx[0] = fmaxf(mx[0], fmaxf(__uint_as_float(sa[c][4 * k]), __uint_as_float(sa[c][4 * k + 1])));
                    mx[1] = fmaxf(mx[1], fmaxf(__uint_as_float(sa[c][4 * k + 2]), __uint_as_float(sa[c][4 * k + 3])));
                    mx[2] = fmaxf(mx[2], fmaxf(__uint_as_float(sb[c][4 * k]), __uint_as_float(sb[c][4 * k + 1])));
                    mx[3] = fmaxf(mx[3], fmaxf(__uint_as_float(sb[c][4 * k + 2]), __uint_as_float(sb[c][4 * k + 3])));
                }
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // the 4 threads of a row hold its 128 columns
                mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 1));
                mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 2));
            }
            bool waited = false;
            if (j == 0) {
#pragma unroll
                for (int k = 0; k < 4; ++k) m_used[k] = mx[k];
            } else {
                // Rescale only when some row's max grew by more than 2^8 in probability
                // units; otherwise keep the stale max (exact, p <= 256 fits bf16 / fp32).
                bool need = false;
#pragma unroll
                for (int k = 0; k < 4; ++k) need |= (mx[k] - m_used[k]) * sl > 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (j - 1) & 1, ab, to, 42));
                    if (!ok) break;
                    waited = true;
                    tc_fence_after();
                    float f[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float mn = fmaxf(m_used[k], mx[k]);
                        f[k] = ex2((m_used[k] - mn) * sl);
                        m_used[k] = mn;
                        l_part[k] *= f[k];
                    }
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t base = half ? tl16 : tl;
                        const float fa = f[2 * half], fb = f[2 * half + 1];
#pragma unroll 1
                        for (int cc = 0; cc < DC; cc += 64) {
                            uint32_t o[32];
                            tmem_ld_16x256b_x8(base + C::O_COL + cc, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int k = 0; k < 8; ++k) {
                                o[4 * k + 0] = __float_as_uint(__uint_as_float(o[4 * k + 0]) * fa);
                                o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * fa);
                                o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * fb);
                                o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * fb);
                            }
                            tmem_st_16x256b_x8(base + C::O_COL + cc, o);
                        }
                    }
                }
            }
            // P = exp2(s * sl - m * sl), packed bf16 pairs for the 16x128b store:
            // rep kk (4 columns) <- pair (8k + 2 quad, +1) of column half c, kk = 8c + k
            float nm[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) nm[k] = -m_used[k] * sl;
            uint32_t pa[32], pb[32];
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int kk = 8 * c + k;
                    const float a0 = ex2(fmaf(__uint_as_float(sa[c][4 * k + 0]), sl, nm[0]));
                    const float a1 = ex2(fmaf(__uint_as_float(sa[c][4 * k + 1]), sl, nm[0]));
                    const float a2 = ex2(fmaf(__uint_as_float(sa[c][4 * k + 2]), sl, nm[1]));
                    const float a3 = ex2(fmaf(__uint_as_float(sa[c][4 * k + 3]), sl, nm[1]));
                    const float b0 = ex2(fmaf(__uint_as_float(sb[c][4 * k + 0]), sl, nm[2]));
                    const float b1 = ex2(fmaf(__uint_as_float(sb[c][4 * k + 1]), sl, nm[2]));
                    const float b2 = ex2(fmaf(__uint_as_float(sb[c][4 * k + 2]), sl, nm[3]));
                    const float b3 = ex2(fmaf(__uint_as_float(sb[c][4 * k + 3]), sl, nm[3]));
                    l_part[0] += a0 + a1;
                    l_part[1] += a2 + a3;
                    l_part[2] += b0 + b1;
                    l_part[3] += b2 + b3;
                    pa[2 * kk + 0] = pack_bf16(a0, a1);
                    pa[2 * kk + 1] = pack_bf16(a2, a3);
                    pb[2 * kk + 0] = pack_bf16(b0, b1);
                    pb[2 * kk + 1] = pack_bf16(b2, b3);
                }
            if (j > 0 && !waited) {  // P_{j-1} must have been consumed before P_j overwrites it
                ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (j - 1) & 1, ab, to, 43));
                if (!ok) break;
                tc_fence_after();
            }
            tmem_st_16x128b_x16(tl + C::P_COL, pa);
            tmem_st_16x128b_x16(tl16 + C::P_COL, pb);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->p_full);
        }

        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (nt - 1) & 1, ab, to, 44) && !ab->flag);
        if (ok) {
            tc_fence_after();
            float inv[4], lt[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                lt[k] = l_part[k];
                lt[k] += __shfl_xor_sync(0xffffffffu, lt[k], 1);
                lt[k] += __shfl_xor_sync(0xffffffffu, lt[k], 2);
                inv[k] = 1.0f / lt[k];
            }
            // O_lat = O / l as hi + lo bf16 parts, K-major SW128 operands in stages
            // (nt+1) % NS and (nt+2) % NS (both drained: every PV has completed)
            uint8_t* ol = stage((nt + 1) % NS);
            uint8_t* ol2 = stage((nt + 2) % NS);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const uint32_t base = half ? tl16 : tl;
                const int r_top = w4 * 32 + half * 16 + (lane >> 2);
                const int r_bot = r_top + 8;
                const float ia = inv[2 * half], ib = inv[2 * half + 1];
#pragma unroll 1
                for (int cc = 0; cc < DC / 64; ++cc) {
                    uint32_t o[32];
                    tmem_ld_16x256b_x8(base + C::O_COL + cc * 64, o);
                    tmem_wait_ld();
                    const int off_top = cc * C::OLAT_ATOM + r_top * 128 + 4 * quad;
                    const int off_bot = cc * C::OLAT_ATOM + r_bot * 128 + 4 * quad;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        uint32_t hi, lo;
                        split_bf16(__uint_as_float(o[4 * k]) * ia, __uint_as_float(o[4 * k + 1]) * ia, hi, lo);
                        const int ot = off_top + ((k ^ (r_top & 7)) << 4);
                        *reinterpret_cast<uint32_t*>(ol + ot) = hi;
                        *reinterpret_cast<uint32_t*>(ol2 + ot) = lo;
                        split_bf16(__uint_as_float(o[4 * k + 2]) * ib, __uint_as_float(o[4 * k + 3]) * ib, hi, lo);
                        const int ob = off_bot + ((k ^ (r_bot & 7)) << 4);
                        *reinterpret_cast<uint32_t*>(ol + ob) = hi;
                        *reinterpret_cast<uint32_t*>(ol2 + ob) = lo;
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->olat_ready);

            if (p.lse != nullptr && quad == 0) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = q0 + w4 * 32 + (lane >> 2) + 8 * k;
                    if (i < p.Nq)
                        p.lse[(size_t(b) * p.Nq + i) * p.H + h] = (m_used[k] * sl + __log2f(lt[k])) * 0.69314718055994531f;
                }
            }

            ok = __all_sync(0xffffffffu, mbar_wait(&bar->out_full, 0, ab, to, 45) && !ab->flag);
            if (ok) {
                tc_fence_after();
                const int i = q0 + w4 * 32 + lane;
                __nv_bfloat16* dst = p.out + ((size_t(b) * p.Nq + i) * p.H + h) * DV;
#pragma unroll 1
                for (int c = 0; c < DV; c += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tl + C::S_COL + c, v);
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
