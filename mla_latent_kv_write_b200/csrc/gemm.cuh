// gemm.cuh -- the plain projections around the latent attention of "VideoMLA:
// Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video Diffusion"
// (arXiv 2605.30351): the query path c^Q = W_dq x (Eq. 3), RMSNorm of c^Q
// (App. D.2), q^nope = W_uq c^Q (Eq. 4) and q^R = W_qr c^Q (Eq. 6, unrotated),
// and the output projection y = W_O [o_1 .. o_H] (the per-head slices of
// Eq. 10-11).
//
// gemm_pair_kernel: C_g [M, N_g] = A [M, K] . B_g [N_g, K]^T for one or two
// column groups g that share A (q^nope and q^R both read the normalised c^Q),
// bf16 operands (both K-major), fp32 accumulation in tensor memory, bf16 or fp32
// C, on CTA pairs (tcgen05 cta_group::2).  A persistent grid of pairs walks the
// 256 x BN output tiles (row tile major, so neighbouring pairs read the same rows
// of A from L2), 192 threads per CTA:
//   warp 0     TMA producer: this CTA's A rows (128 x 64) and half of the B tile
//              (BN/2 x 64) per stage, 128B swizzle (rows past M or N read zeros)
//   warp 1     TMEM owner; on rank 0, tcgen05.mma.cta_group::2 issuer (M 256,
//              N BN, K 16 steps); two accumulators, so the next tile's MMAs run
//              while the epilogues drain this one
//   warps 2-5  epilogue: one TMEM lane (row of C) per thread, 16-byte stores
//              of the columns below N; optionally a per-row sum of squares
//              (atomically added), a per-column scale and a per-row 1 / rms
//              scale, which together carry the query path's RMSNorm
#pragma once

#include "ptx.cuh"

namespace vmla {

struct GemmParams {
    int M, K;
    int n_groups;         // 1 or 2 column groups
    int N[2];             // columns of each group
    int n_tiles[2];       // BN-wide column tiles of each group
    int m_tiles, tiles;   // row tiles; all tiles
    void* C[2];           // [M, ldc] bf16 or fp32, row-major
    int ldc[2];           // elements
    uint64_t timeout_ns;
    // optional epilogue work (RMSNorm split across two GEMMs): row_ss[t M + row] = sum
    // of the row's squared fp32 outputs in column tile t (one column group; every
    // (row, tile) written once, so no zeroing and no atomics); column c scaled by
    // col_scale[c]; every row scaled by 1 / sqrt(ms / rms_dim + rms_eps), ms the sum
    // of row_ss_in[k M + row] over k < ss_parts, in order
    float* row_ss;
    const float* col_scale;
    const float* row_ss_in;
    int ss_parts;
    int rms_dim;
    float rms_eps;
};

// Tile index -> (row tile, column group, first column in the group).
__device__ __forceinline__ void gemm_tile(const GemmParams& p, int tile, int BN, int& m0, int& g, int& n0) {
    const int per_row = p.n_tiles[0] + p.n_tiles[1];
    const int mt = tile / per_row, nt = tile - mt * per_row;
    m0 = mt * 128;
    g = nt < p.n_tiles[0] ? 0 : 1;
    n0 = (g == 0 ? nt : nt - p.n_tiles[0]) * BN;
}

// gemm_pair_kernel: the same product on CTA pairs.  A cluster of 2 CTAs owns a
// 256 x BN output tile: CTA r of the pair loads rows [128 r, 128 r + 128) of the
// A tile and rows [r BN/2, (r + 1) BN/2) of the B tile, and rank 0 issues
// tcgen05.mma.cta_group::2 (M 256, N BN), which reads both CTAs' shared memory
// and leaves each CTA's 128 rows of D in its own tensor memory.  Each SM thus
// pulls half of B per output instead of all of it.  Both CTAs' loads complete
// on rank 0's stage barrier; rank 0's commits arrive on both CTAs' barriers;
// both CTAs' epilogues free an accumulator on rank 0's barrier.
template <int BN_, bool F32OUT_>
struct GemmPairCfg {
    static constexpr int BM = 128, BN = BN_, BNH = BN_ / 2, BK = 64;
    static constexpr bool F32OUT = F32OUT_;
    static constexpr int A_BYTES = BM * BK * 2, B_BYTES = BNH * BK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NS = (232448 - 2048) / STAGE > 8 ? 8 : (232448 - 2048) / STAGE;
    static constexpr int SMEM = NS * STAGE + 1024 + 256;
    static constexpr int THREADS = 192;
    static constexpr int TMEM_COLS = 2 * BN;  // two accumulators of BN columns
    static_assert(BN == 128 || BN == 256, "tile width");
    static_assert(STAGE % 1024 == 0 && SMEM <= 232448, "shared memory");
};

template <class C>
__global__ void __launch_bounds__(192, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                     const __grid_constant__ CUtensorMap tm_b1, const GemmParams p) {
    constexpr int BN = C::BN, BNH = C::BNH, BK = C::BK, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * C::STAGE);  // rank 0's are used
    uint64_t* empty = full + NS;
    uint64_t* acc_full = empty + NS;     // [2]
    uint64_t* acc_empty = acc_full + 2;  // [2], rank 0's are used
    uint64_t* done = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const int pair = int(blockIdx.x) >> 1, P = int(gridDim.x) >> 1;
    const int k_chunks = p.K / BK;
    const uint64_t to = p.timeout_ns;
    griddep_launch_dependents();  // the grid is persistent: all of it is resident from the start

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 8);  // 4 epilogue warps of each CTA
        }
        mbar_init(done, 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or byte count
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Launched programmatically: the set-up above overlaps the previous kernel's
    // tail; no thread touches global memory before that kernel has finished.
    griddep_wait();
    auto stage_a = [&](int s) { return smem + s * C::STAGE; };
    auto stage_b = [&](int s) { return smem + s * C::STAGE + C::A_BYTES; };

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b0);
            if (p.n_groups > 1) tma_prefetch_desc(&tm_b1);
            const uint32_t full0 = mapa_shared(smem_u32(full), 0);  // rank 0's stage barriers
            int it = 0;
            bool ok = true;
            for (int tile = pair; tile < p.tiles && ok; tile += P) {
                int m0, g, n0;
                gemm_tile(p, tile, BN, m0, g, n0);  // m0: first row of the pair's 256
                m0 = 2 * m0 + int(rank) * 128;
                const CUtensorMap* tb = g == 0 ? &tm_b0 : &tm_b1;
                for (int kc = 0; kc < k_chunks; ++kc, ++it) {
                    const int s = it % NS;
                    if (it >= NS && !mbar_wait_cl(&empty[s], ((it / NS) - 1) & 1, ab, to, 54)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * C::STAGE);
                    tma_load_2d_pair(stage_a(s), &tm_a, full0 + 8u * s, kc * BK, m0);
                    tma_load_2d_pair(stage_b(s), tb, full0 + 8u * s, kc * BK, n0 + int(rank) * BNH);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(256, BN, false, false);
            bool ok = true;
            int it = 0, j = 0;
            for (int tile = pair; tile < p.tiles && ok; tile += P, ++j) {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_cl(&acc_empty[buf], ((j >> 1) - 1) & 1, ab, to, 55)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + uint32_t(buf * BN);
                for (int kc = 0; kc < k_chunks; ++kc, ++it) {
                    const int s = it % NS;
                    if (!mbar_wait_cl(&full[s], (it / NS) & 1, ab, to, 56)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = smem_u32(stage_a(s)), b = smem_u32(stage_b(s));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_ss_pair(acc, sdesc(a + kk * 32, 16, 1024, SW128), sdesc(b + kk * 32, 16, 1024, SW128),
                                     idesc, (kc | kk) != 0);
                    umma_commit_pair_mc(&empty[s], 0x3);  // both CTAs may refill stage s
                }
                if (ok) umma_commit_pair_mc(&acc_full[buf], 0x3);
            }
            umma_commit_pair_mc(done, 0x1);
            mbar_wait_drain(done, 0, to);  // no MMA may be in flight at teardown
        }
    } else {
        // epilogue: TMEM lane r = row m0 + r of this CTA's half of the pair tile
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
        int j = 0;
        for (int tile = pair; tile < p.tiles; tile += P, ++j) {
            int m0, g, n0;
            gemm_tile(p, tile, BN, m0, g, n0);
            m0 = 2 * m0 + int(rank) * 128;
            const int buf = j & 1;
            const bool go = __all_sync(0xffffffffu, mbar_wait_cl(&acc_full[buf], (j >> 1) & 1, ab, to, 57));
            if (!go || ab->flag) break;  // warps leave independently: no barrier among them follows
            tc_fence_after();
            const uint32_t trow = tmem + uint32_t(buf * BN) + (uint32_t(quarter * 32) << 16);
            const int row = m0 + r;
            const int N = g == 0 ? p.N[0] : p.N[1], ldc = g == 0 ? p.ldc[0] : p.ldc[1];
            void* const Cg = g == 0 ? p.C[0] : p.C[1];
            float rscale = 1.0f;
            if (p.row_ss_in != nullptr && row < p.M) {
                float ms = 0.f;
                for (int k = 0; k < p.ss_parts; ++k) ms += __ldg(p.row_ss_in + size_t(k) * p.M + row);
                rscale = rsqrtf(ms / float(p.rms_dim) + p.rms_eps);
            }
            float ss = 0.f;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(trow + c, v);
                tmem_wait_ld();
                if (p.row_ss != nullptr) {  // columns past N are zeros (B rows past N read zeros)
#pragma unroll
                    for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), ss);
                }
                if (p.col_scale != nullptr || p.row_ss_in != nullptr) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4) {
                        float4 cs = make_float4(1.f, 1.f, 1.f, 1.f);
                        if (p.col_scale != nullptr && n0 + c + e + 4 <= N)
                            cs = __ldg(reinterpret_cast<const float4*>(p.col_scale + n0 + c + e));
                        v[e + 0] = __float_as_uint(__uint_as_float(v[e + 0]) * cs.x * rscale);
                        v[e + 1] = __float_as_uint(__uint_as_float(v[e + 1]) * cs.y * rscale);
                        v[e + 2] = __float_as_uint(__uint_as_float(v[e + 2]) * cs.z * rscale);
                        v[e + 3] = __float_as_uint(__uint_as_float(v[e + 3]) * cs.w * rscale);
                    }
                }
                if (row < p.M) {
                    if constexpr (C::F32OUT) {
                        float* dst = static_cast<float*>(Cg) + size_t(row) * ldc + n0 + c;
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            if (n0 + c + e + 4 <= N)
                                *reinterpret_cast<float4*>(dst + e) =
                                    make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                    } else {
                        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(Cg) + size_t(row) * ldc + n0 + c;
#pragma unroll
                        for (int e = 0; e < 32; e += 8)
                            if (n0 + c + e + 8 <= N)
                                *reinterpret_cast<uint4*>(dst + e) = make_uint4(
                                    pack_bf16(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                                    pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                                    pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                                    pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
                    }
                }
            }
            if (p.row_ss != nullptr && row < p.M) p.row_ss[size_t(n0 / BN) * p.M + row] = ss;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {  // the accumulator may take tile j + 2 (rank 0's barrier counts both CTAs)
                if (rank == 0) mbar_arrive(&acc_empty[buf]);
                else mbar_arrive_remote(acc_empty0 + 8u * buf);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // rank 0's MMAs no longer read this CTA's shared memory; no arrive is in flight
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::TMEM_COLS);
    }
}

}  // namespace vmla
