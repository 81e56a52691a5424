// gemm.cuh -- the plain projections around the latent attention of "VideoMLA:
// Low-Rank Latent KV Cache for Minute-Scale Autoregressive Video Diffusion"
// (arXiv 2605.30351): the query path c^Q = W_dq x (Eq. 3), RMSNorm of c^Q
// (App. D.2), q^nope = W_uq c^Q (Eq. 4) and q^R = W_qr c^Q (Eq. 6, unrotated),
// and the output projection y = W_O [o_1 .. o_H] (the per-head slices of
// Eq. 10-11).
//
// gemm_kernel: C_g [M, N_g] = A [M, K] . B_g [N_g, K]^T for one or two column
// groups g that share A (q^nope and q^R both read the normalised c^Q), bf16
// operands (both K-major), fp32 accumulation in tensor memory, bf16 or fp32 C.
// A persistent grid of one CTA per SM walks the 128 x BN output tiles (row tile
// major, so neighbouring CTAs read the same rows of A from L2), 192 threads:
//   warp 0     TMA producer: A tile 128 x 64 and B tile BN x 64 per stage,
//              128B swizzle (rows past M or N read zeros)
//   warp 1     tcgen05.mma issuer (M 128, N BN, K 16 steps) and TMEM owner;
//              two accumulators, so the next tile's MMAs run while the
//              epilogue drains this one
//   warps 2-5  epilogue: one TMEM lane (row of C) per thread, 16-byte stores
//              of the columns below N
// rms_norm_rows_kernel: one warp per row of an fp32 [M, D] matrix, bf16 output
// g * v / sqrt(mean(v^2) + eps).
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
};

template <int BN_, bool F32OUT_>
struct GemmCfg {
    static constexpr int BM = 128, BN = BN_, BK = 64;
    static constexpr bool F32OUT = F32OUT_;
    static constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NS = (232448 - 2048) / STAGE > 8 ? 8 : (232448 - 2048) / STAGE;  // pipeline stages
    static constexpr int SMEM = NS * STAGE + 1024 + 256;
    static constexpr int THREADS = 192;
    static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
    static_assert(BN == 128 || BN == 256, "tile width");
    static_assert(SMEM <= 232448, "shared memory");
};

// Tile index -> (row tile, column group, first column in the group).
__device__ __forceinline__ void gemm_tile(const GemmParams& p, int tile, int BN, int& m0, int& g, int& n0) {
    const int per_row = p.n_tiles[0] + p.n_tiles[1];
    const int mt = tile / per_row, nt = tile - mt * per_row;
    m0 = mt * 128;
    g = nt < p.n_tiles[0] ? 0 : 1;
    n0 = (g == 0 ? nt : nt - p.n_tiles[0]) * BN;
}

template <class C>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                const __grid_constant__ CUtensorMap tm_b1, const GemmParams p) {
    constexpr int BM = C::BM, BN = C::BN, BK = C::BK, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * C::STAGE);
    uint64_t* empty = full + NS;
    uint64_t* acc_full = empty + NS;     // [2]
    uint64_t* acc_empty = acc_full + 2;  // [2]
    uint64_t* done = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();
    const int G = gridDim.x;
    const int k_chunks = p.K / BK;
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(done, 1);
        ab->flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto stage_a = [&](int s) { return smem + s * C::STAGE; };
    auto stage_b = [&](int s) { return smem + s * C::STAGE + C::A_BYTES; };

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b0);
            if (p.n_groups > 1) tma_prefetch_desc(&tm_b1);
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.tiles && ok; tile += G) {
                int m0, g, n0;
                gemm_tile(p, tile, BN, m0, g, n0);
                const CUtensorMap* tb = g == 0 ? &tm_b0 : &tm_b1;
                for (int kc = 0; kc < k_chunks; ++kc, ++it) {
                    const int s = it % NS;
                    if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1, ab, to, 50)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_2d(stage_a(s), &tm_a, &full[s], kc * BK, m0);
                    tma_load_2d(stage_b(s), tb, &full[s], kc * BK, n0);
                }
            }
            if (!ok || ab->flag) {  // let the copies still in flight land before the CTA exits
                for (int j = it - NS < 0 ? 0 : it - NS; j < it; ++j)
                    mbar_wait_drain(&full[j % NS], (j / NS) & 1, to);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
            bool ok = true;
            int it = 0, j = 0;
            for (int tile = blockIdx.x; tile < p.tiles && ok; tile += G, ++j) {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait(&acc_empty[buf], ((j >> 1) - 1) & 1, ab, to, 53)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + uint32_t(buf * BN);
                for (int kc = 0; kc < k_chunks; ++kc, ++it) {
                    const int s = it % NS;
                    if (!mbar_wait(&full[s], (it / NS) & 1, ab, to, 51)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = smem_u32(stage_a(s)), b = smem_u32(stage_b(s));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_ss(acc, sdesc(a + kk * 32, 16, 1024, SW128), sdesc(b + kk * 32, 16, 1024, SW128), idesc,
                                (kc | kk) != 0);
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(&acc_full[buf]);
            }
            umma_commit(done);
            mbar_wait_drain(done, 0, to);  // no MMA may be in flight at teardown
        }
    } else {
        // epilogue: TMEM lane r = row m0 + r of the tile
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        int j = 0;
        for (int tile = blockIdx.x; tile < p.tiles; tile += G, ++j) {
            int m0, g, n0;
            gemm_tile(p, tile, BN, m0, g, n0);
            const int buf = j & 1;
            const bool go = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (j >> 1) & 1, ab, to, 52));
            if (!go || ab->flag) break;  // warps leave independently: no barrier among them follows
            tc_fence_after();
            const uint32_t trow = tmem + uint32_t(buf * BN) + (uint32_t(quarter * 32) << 16);
            const int row = m0 + r;
            const int N = g == 0 ? p.N[0] : p.N[1], ldc = g == 0 ? p.ldc[0] : p.ldc[1];
            void* const Cg = g == 0 ? p.C[0] : p.C[1];
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(trow + c, v);
                tmem_wait_ld();
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
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);  // the accumulator may take tile j + 2
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// out[m, :] = bf16(g * in[m, :] / sqrt(mean(in[m, :]^2) + eps)), D % 4 == 0; one warp per row.
__global__ void __launch_bounds__(256) rms_norm_rows_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                                            const float* __restrict__ gamma, int M, int D, float eps) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= M) return;
    const float* src = in + size_t(row) * D;
    float ss = 0.f;
    for (int c = lane * 4; c < D; c += 128) {
        const float4 v = *reinterpret_cast<const float4*>(src + c);
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float scale = rsqrtf(ss / float(D) + eps);
    __nv_bfloat16* dst = out + size_t(row) * D;
    for (int c = lane * 4; c < D; c += 128) {
        const float4 v = *reinterpret_cast<const float4*>(src + c);
        float g0 = 1.f, g1 = 1.f, g2 = 1.f, g3 = 1.f;
        if (gamma != nullptr) {
            const float4 g = *reinterpret_cast<const float4*>(gamma + c);
            g0 = g.x; g1 = g.y; g2 = g.z; g3 = g.w;
        }
        *reinterpret_cast<uint2*>(dst + c) =
            make_uint2(pack_bf16(v.x * scale * g0, v.y * scale * g1), pack_bf16(v.z * scale * g2, v.w * scale * g3));
    }
}

}  // namespace vmla
