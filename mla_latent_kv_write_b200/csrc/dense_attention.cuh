// dense_attention.cuh -- the dense multi-head attention that "VideoMLA: Low-Rank
// Latent KV Cache for Minute-Scale Autoregressive Video Diffusion" (arXiv
// 2605.30351) compares against (App. C.1: every token caches per-head keys and
// values, 2 n_h d_h = 3072 scalars per token and layer, against the 224 of the
// latent cache), as a baseline kernel of this library: the same window, the same
// 3D-RoPE positions and the same softmax as the latent kernel, over keys
// k_h = [k^nope_h | RoPE3D(k^R)] and values v_h (d_h = 128 each) read per head
// from a dense cache, with no absorption and no W_uv epilogue.
//
// One CTA per (128-query tile, head, batch element), 352 threads, the pipeline
// of the latent kernel:
//   warp 0     TMA producer: K and V tiles of 128 keys (two 64-column SW128
//              blocks each) into a 3-stage ring
//   warp 1     tensor-memory owner; S = Q K^T (Q in TMEM, 8 bf16 K-steps)
//   warps 2-9  softmax, 16 query rows each: q = [q^nope | RoPE3D(q^R)] -> bf16 Q
//              in TMEM, fp32 online softmax, P -> TMEM, O rescale, O / l -> out
//   warp 10    O += P V (V read MN-major from its tile)
// Tensor memory: O [0, 128)  S [128, 256)  P (bf16 pairs) [256, 320)  Q [320, 384).
#pragma once

#include "ptx.cuh"

namespace vmla {

struct DenseParams {
    int Nq, Nk, H;
    int T_f, grid_w;
    int q_first;          // window index of query 0 (the queries are the newest Nq keys' positions)
    int n_t, n_h;         // rope pairs of the t and h axes (w takes the rest)
    float omega[32];      // rope frequency of each pair
    float scale_log2;     // log2(e) / sqrt(d_h)
    const __nv_bfloat16* q_nope;  // [B, Nq, H, DN]
    const __nv_bfloat16* q_rope;  // [B, Nq, H, DR], unrotated
    __nv_bfloat16* out;           // [B, Nq, H, 128]
    uint64_t timeout_ns;
};

// K and V of the window in logical order: (128, H, Nk, B), box (64, 1, 128, 1), 128B swizzle.
struct DenseMaps {
    CUtensorMap k, v;
};

template <int DN_, int DR_>
struct DenseCfg {
    static constexpr int DN = DN_, DR = DR_, DH = DN_ + DR_, DV = 128;
    static constexpr int BM = 128, BK = 128, NS = 3;
    static constexpr int ATOM = BK * 128;             // one 64-column block of a K or V tile
    static constexpr int STAGE = 4 * ATOM;            // K (2 blocks) + V (2 blocks)
    static constexpr int O_COL = 0, S_COL = DV, P_COL = DV + BK, Q_COL = DV + BK + BK / 2;
    static constexpr int SMEM = NS * STAGE + 2048;
    static constexpr int SM_WARPS = 8;
    static constexpr int THREADS = 32 * (3 + SM_WARPS);
    static_assert(DH == 128 && DN % 8 == 0 && DR % 8 == 0, "a 128-wide head of 8-column groups");
    static_assert(Q_COL + DH / 2 <= 512 && SMEM <= 232448, "budgets");
};

struct DenseBarriers {
    uint64_t full[3], empty[3];
    uint64_t q_ready, s_full, s_free, p_full, pv_done, drain, drain2;
    uint32_t tmem_base;
    AbortState ab;
};

// Rotate the pair (x, y) by theta and pack it as bf16x2 (the dense cache is bf16).
__device__ __forceinline__ uint32_t rotate_pair_bf16(uint32_t v_bf16x2, float theta) {
    float sn, cs;
    sincosf(theta, &sn, &cs);
    const float x = bf16_lo(v_bf16x2), y = bf16_hi(v_bf16x2);
    return pack_bf16(x * cs - y * sn, x * sn + y * cs);
}

template <class C>
__global__ void __launch_bounds__(352, 1) dense_attention_kernel(const __grid_constant__ DenseMaps maps,
                                                                 const DenseParams p) {
    constexpr int DN = C::DN, DR = C::DR, DH = C::DH, DV = C::DV, BM = C::BM, BK = C::BK, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DenseBarriers* bar = reinterpret_cast<DenseBarriers*>(smem + NS * C::STAGE);
    AbortState* ab = &bar->ab;
    auto stage = [&](int s) { return smem + s * C::STAGE; };

    const int warp = warp_id(), lane = lane_id();
    const int h = blockIdx.y, b = blockIdx.z;
    const int q0 = blockIdx.x * BM;
    const int nt = (p.Nk + BK - 1) / BK;
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bar->full[s], 1);
            mbar_init(&bar->empty[s], 1);
        }
        mbar_init(&bar->q_ready, C::SM_WARPS);
        mbar_init(&bar->s_full, 1);
        mbar_init(&bar->s_free, C::SM_WARPS);
        mbar_init(&bar->p_full, C::SM_WARPS);
        mbar_init(&bar->pv_done, 1);
        mbar_init(&bar->drain, 1);
        mbar_init(&bar->drain2, 1);
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
            tma_prefetch_desc(&maps.k);
            tma_prefetch_desc(&maps.v);
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int s = j % NS;
                if (j >= NS && !mbar_wait(&bar->empty[s], ((j / NS) - 1) & 1, ab, to, 60)) break;
                mbar_arrive_expect_tx(&bar->full[s], C::STAGE);
                for (int a = 0; a < 2; ++a) {
                    tma_load_4d(stage(s) + a * C::ATOM, &maps.k, &bar->full[s], a * 64, h, j * BK, b);
                    tma_load_4d(stage(s) + (2 + a) * C::ATOM, &maps.v, &bar->full[s], a * 64, h, j * BK, b);
                }
                issued = j + 1;
            }
            if (ab->flag) {  // let this CTA's copies land before it exits
                for (int j = issued > NS ? issued - NS : 0; j < issued; ++j)
                    mbar_wait_drain(&bar->full[j % NS], (j / NS) & 1, to);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ S issuer
        if (lane == 0) {
            bool ok = mbar_wait(&bar->q_ready, 0, ab, to, 61);
            constexpr uint32_t id_s = idesc_bf16_f32(128, BK, false, false);
            for (int j = 0; ok && j < nt; ++j) {
                const int s = j % NS;
                ok = mbar_wait(&bar->full[s], (j / NS) & 1, ab, to, 62);
                if (ok && j > 0) ok = mbar_wait(&bar->s_free, (j - 1) & 1, ab, to, 63);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(stage(s));
#pragma unroll
                for (int k = 0; k < DH / 16; ++k)
                    umma_ts(tmem + C::S_COL, tmem + C::Q_COL + k * 8,
                            sdesc(st + (k / 4) * C::ATOM + (k % 4) * 32, 16, 1024, SW128), id_s, k > 0);
                umma_commit(&bar->s_full);
            }
            if (!ok) {  // no MMA may still run when the tensor memory is released
                umma_commit(&bar->drain);
                mbar_wait_drain(&bar->drain, 0, to);
            }
        }
    } else if (warp == 2 + C::SM_WARPS) {
        // ------------------------------------------------------------ PV issuer
        if (lane == 0) {
            constexpr uint32_t id_pv = idesc_bf16_f32(128, DV, false, true);
            bool ok = true;
            for (int jj = 0; ok && jj < nt; ++jj) {
                const int sp = jj % NS;
                ok = mbar_wait(&bar->p_full, jj & 1, ab, to, 64);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sv = smem_u32(stage(sp)) + 2 * C::ATOM;
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    umma_ts(tmem + C::O_COL, tmem + C::P_COL + k * 8, sdesc(sv + k * 2048, C::ATOM, 1024, SW128),
                            id_pv, (jj > 0 || k > 0));
                umma_commit(&bar->empty[sp]);
                umma_commit(&bar->pv_done);
            }
            umma_commit(&bar->drain2);
            mbar_wait_drain(&bar->drain2, 0, to);
        }
    } else {
        // ------------------------------------------------------------ softmax / epilogue
        // warps 2-9; warps 2-5 own lanes 0-15 of their TMEM quadrant, warps 6-9 lanes
        // 16-31, so every query row belongs to exactly one warp.
        const int w4 = warp & 3;
        const int half = (warp - 2) >> 2;
        const int quad = lane & 3;
        const uint32_t tq = tmem + (uint32_t(w4 * 32) << 16);
        const uint32_t tb = tq + (uint32_t(half * 16) << 16);
        const float sl = p.scale_log2;

        // prologue: Q = bf16 [q^nope | RoPE3D(q^R)], one row per thread; the two warps
        // of a quadrant take alternate 32-column chunks
        {
            const int r = w4 * 32 + lane;
            const int i = q0 + r;
            const bool live = i < p.Nq;
            const uint4* qn = reinterpret_cast<const uint4*>(p.q_nope + ((size_t(b) * p.Nq + (live ? i : 0)) * p.H + h) * DN);
            const uint4* qr = reinterpret_cast<const uint4*>(p.q_rope + ((size_t(b) * p.Nq + (live ? i : 0)) * p.H + h) * DR);
            const int L = p.q_first + i;
            const int tq_ = L / p.T_f;
            const int pq = L - tq_ * p.T_f;
            const int hq = pq / p.grid_w, wq = pq - (pq / p.grid_w) * p.grid_w;
#pragma unroll 1
            for (int c = half; c < DH / 32; c += 2) {
                uint32_t pk[16];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int col = 32 * c + 8 * g;
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (live) {
                        if (col < DN) {
                            v = __ldg(qn + col / 8);
                        } else {
                            const int pr = (col - DN) / 2;  // first rope pair of the group
                            const uint4 u = __ldg(qr + (col - DN) / 8);
                            v.x = rotate_pair_bf16(u.x, float(pr + 0 < p.n_t ? tq_ : pr + 0 < p.n_t + p.n_h ? hq : wq) * p.omega[pr + 0]);
                            v.y = rotate_pair_bf16(u.y, float(pr + 1 < p.n_t ? tq_ : pr + 1 < p.n_t + p.n_h ? hq : wq) * p.omega[pr + 1]);
                            v.z = rotate_pair_bf16(u.z, float(pr + 2 < p.n_t ? tq_ : pr + 2 < p.n_t + p.n_h ? hq : wq) * p.omega[pr + 2]);
                            v.w = rotate_pair_bf16(u.w, float(pr + 3 < p.n_t ? tq_ : pr + 3 < p.n_t + p.n_h ? hq : wq) * p.omega[pr + 3]);
                        }
                    }
                    pk[4 * g + 0] = v.x;
                    pk[4 * g + 1] = v.y;
                    pk[4 * g + 2] = v.z;
                    pk[4 * g + 3] = v.w;
                }
                tmem_st_32x32b_x16(tq + C::Q_COL + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->q_ready);
        }

        // main loop.  16x256b layout: this thread holds rows
        //   R0 = w4*32 + half*16 + lane/4 and R1 = R0 + 8, 32 columns of each
        //   (columns 8k + 2 quad + {0, 1} of each 64-column half of the tile).
        bool ok = true;
        float m_used[2] = {0.f, 0.f}, l_part[2] = {0.f, 0.f};
        for (int j = 0; ok && j < nt; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->s_full, j & 1, ab, to, 65));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[2][32];
#pragma unroll
            for (int c = 0; c < 2; ++c) tmem_ld_16x256b_x8(tb + C::S_COL + 64 * c, sv[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->s_free);

            const int valid = min(BK, p.Nk - j * BK);
            if (valid < BK) {  // ragged last tile: mask the missing keys
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
#pragma unroll
                        for (int e = 0; e < 2; ++e)
                            if (64 * c + 8 * k + 2 * quad + e >= valid)
                                sv[c][4 * k + e] = sv[c][4 * k + 2 + e] = 0xff800000u;  // -inf
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    mx[0] = fmaxf(mx[0], fmaxf(__uint_as_float(sv[c][4 * k]), __uint_as_float(sv[c][4 * k + 1])));
                    mx[1] = fmaxf(mx[1], fmaxf(__uint_as_float(sv[c][4 * k + 2]), __uint_as_float(sv[c][4 * k + 3])));
                }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 1));
                mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 2));
            }
            bool waited = false;
            if (j == 0) {
                m_used[0] = mx[0];
                m_used[1] = mx[1];
            } else {
                // rescale only when some row's max grew by more than 2^8 in probability units
                const bool need = (mx[0] - m_used[0]) * sl > 8.0f || (mx[1] - m_used[1]) * sl > 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (j - 1) & 1, ab, to, 66));
                    if (!ok) break;
                    waited = true;
                    tc_fence_after();
                    float f[2];
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const float mn = fmaxf(m_used[k], mx[k]);
                        f[k] = ex2((m_used[k] - mn) * sl);
                        m_used[k] = mn;
                        l_part[k] *= f[k];
                    }
#pragma unroll 1
                    for (int cc = 0; cc < DV; cc += 64) {
                        uint32_t o[32];
                        tmem_ld_16x256b_x8(tb + C::O_COL + cc, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            o[4 * k + 0] = __float_as_uint(__uint_as_float(o[4 * k + 0]) * f[0]);
                            o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * f[0]);
                            o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * f[1]);
                            o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * f[1]);
                        }
                        tmem_st_16x256b_x8(tb + C::O_COL + cc, o);
                    }
                }
            }
            // P = exp2(s * sl - m * sl) as bf16 pairs for the 16x128b store
            const float2 sl2 = make_float2(sl, sl);
            const float2 nm0 = make_float2(-m_used[0] * sl, -m_used[0] * sl);
            const float2 nm1 = make_float2(-m_used[1] * sl, -m_used[1] * sl);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
            uint32_t pa[32];
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int kk = 8 * c + k;
                    const float2 x01 = __ffma2_rn(
                        make_float2(__uint_as_float(sv[c][4 * k + 0]), __uint_as_float(sv[c][4 * k + 1])), sl2, nm0);
                    const float2 x23 = __ffma2_rn(
                        make_float2(__uint_as_float(sv[c][4 * k + 2]), __uint_as_float(sv[c][4 * k + 3])), sl2, nm1);
                    const float2 e01 = make_float2(ex2(x01.x), ex2(x01.y));
                    const float2 e23 = make_float2(ex2(x23.x), ex2(x23.y));
                    acc0 = __fadd2_rn(acc0, e01);
                    acc1 = __fadd2_rn(acc1, e23);
                    pa[2 * kk + 0] = pack_bf16(e01.x, e01.y);
                    pa[2 * kk + 1] = pack_bf16(e23.x, e23.y);
                }
            l_part[0] += acc0.x + acc0.y;
            l_part[1] += acc1.x + acc1.y;
            if (j > 0 && !waited) {  // P_{j-1} must have been consumed before P_j overwrites it
                ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (j - 1) & 1, ab, to, 67));
                if (!ok) break;
                tc_fence_after();
            }
            tmem_st_16x128b_x16(tb + C::P_COL, pa);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->p_full);
        }

        // epilogue: out = O / l, bf16, straight from tensor memory
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (nt - 1) & 1, ab, to, 68) && !ab->flag);
        if (ok) {
            tc_fence_after();
            float inv[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                float l = l_part[k];
                l += __shfl_xor_sync(0xffffffffu, l, 1);
                l += __shfl_xor_sync(0xffffffffu, l, 2);
                inv[k] = 1.0f / l;
            }
            const int r_top = w4 * 32 + half * 16 + (lane >> 2);
            const int i_top = q0 + r_top, i_bot = i_top + 8;
#pragma unroll 1
            for (int cc = 0; cc < DV; cc += 64) {
                uint32_t o[32];
                tmem_ld_16x256b_x8(tb + C::O_COL + cc, o);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int col = cc + 8 * k + 2 * quad;
                    if (i_top < p.Nq)
                        *reinterpret_cast<uint32_t*>(p.out + ((size_t(b) * p.Nq + i_top) * p.H + h) * DV + col) =
                            pack_bf16(__uint_as_float(o[4 * k + 0]) * inv[0], __uint_as_float(o[4 * k + 1]) * inv[0]);
                    if (i_bot < p.Nq)
                        *reinterpret_cast<uint32_t*>(p.out + ((size_t(b) * p.Nq + i_bot) * p.H + h) * DV + col) =
                            pack_bf16(__uint_as_float(o[4 * k + 2]) * inv[1], __uint_as_float(o[4 * k + 3]) * inv[1]);
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
