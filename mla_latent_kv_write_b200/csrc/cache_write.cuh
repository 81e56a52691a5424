// cache_write.cuh -- latent ring-cache write of "VideoMLA: Low-Rank Latent KV
// Cache for Minute-Scale Autoregressive Video Diffusion" (arXiv 2605.30351):
// [c | k^R] = x [W_dkv ; W_kr]^T (Sec. 3.1 Eq. 1, Sec. 3.2 Eq. 5), RMSNorm of
// the latent part (App. D.2), bf16 rows written into the FIFO frame ring
// (App. D.4).  k^R is stored unrotated and unnormalised.
//
// One CTA per (128-token tile, batch element); 192 threads:
//   warp 0     TMA producer (x tile 128 x 64 and W tile N x 64 per stage)
//   warp 1     tcgen05.mma issuer (M = 128, N = d_c + d_rope, K = 16 steps)
//              and tensor-memory owner
//   warps 2-5  epilogue: one TMEM lane (token) per thread, RMSNorm in fp32,
//              bf16 RNE, 16-byte stores into the ring rows
#pragma once

#include "ptx.cuh"

namespace vmla {

struct CacheWriteParams {
    int n_tok;            // tokens per batch element in this call
    int d_model;
    int T_f;              // tokens per latent frame
    int slots;            // ring capacity in frames
    int first_slot;       // slot of frame 0 of the chunk
    int normalize;        // 0: cache the raw down-projection
    float eps;
    const float* gamma;   // [d_c] or null (unit gain)
    __nv_bfloat16* cache; // [B, slots * T_f, d_c + d_rope]
    uint64_t timeout_ns;
};

template <int DC, int DR>
struct CacheWriteCfg {
    static constexpr int N = DC + DR;                 // cached scalars per token
    static constexpr int BM = 128;                    // tokens per CTA
    static constexpr int BKK = 64;                    // K elements per stage (one 128-B swizzle row)
    static constexpr int N_MMA = N <= 256 ? 1 : 2;    // MMA column chunks
    static constexpr int N_CHUNK = N / N_MMA;
    static constexpr int NS = N <= 256 ? 4 : 3;       // pipeline stages
    static constexpr int X_BYTES = BM * BKK * 2;
    static constexpr int W_BYTES = N * BKK * 2;
    static constexpr int STAGE = X_BYTES + W_BYTES;
    static constexpr int WBOX = DC <= 192 ? DC : 192; // rows per W_dkv TMA box
    static constexpr int TMEM_COLS = N <= 256 ? 256 : 512;
    static constexpr int SMEM = NS * STAGE + 1024 + 256;
    static constexpr int THREADS = 192;
    static_assert(N % 16 == 0 && N_CHUNK % 16 == 0 && N_CHUNK <= 256, "MMA N");
    static_assert(DC % 32 == 0 && DR % 16 == 0 && DC % WBOX == 0, "widths");
    static_assert((N * 2) % 16 == 0, "cache row must be 16-byte aligned");
};

template <int DC, int DR>
__global__ void __launch_bounds__(192, 1)
    cache_write_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wdkv,
                       const __grid_constant__ CUtensorMap tm_wkr, const CacheWriteParams p) {
    using C = CacheWriteCfg<DC, DR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NS * C::STAGE);
    uint64_t* empty = full + C::NS;
    uint64_t* done = empty + C::NS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();
    const int row0 = blockIdx.x * C::BM;
    const int b = blockIdx.y;
    const int k_chunks = p.d_model / C::BKK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
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

    auto stage_x = [&](int s) { return smem + s * C::STAGE; };
    auto stage_w = [&](int s) { return smem + s * C::STAGE + C::X_BYTES; };

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_wdkv);
            tma_prefetch_desc(&tm_wkr);
            int issued = 0;
            for (int kc = 0; kc < k_chunks; ++kc) {
                const int s = kc % C::NS;
                if (kc >= C::NS && !mbar_wait(&empty[s], ((kc / C::NS) - 1) & 1, ab, p.timeout_ns, 1)) break;
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                tma_load_3d(stage_x(s), &tm_x, &full[s], kc * C::BKK, row0, b);
                for (int r = 0; r < DC; r += C::WBOX)
                    tma_load_2d(stage_w(s) + r * 128, &tm_wdkv, &full[s], kc * C::BKK, r);
                tma_load_2d(stage_w(s) + DC * 128, &tm_wkr, &full[s], kc * C::BKK, 0);
                issued = kc + 1;
            }
            if (ab->flag) {  // let the copies still in flight land before the CTA exits
                for (int kc = issued - C::NS < 0 ? 0 : issued - C::NS; kc < issued; ++kc)
                    mbar_wait_drain(&full[kc % C::NS], (kc / C::NS) & 1, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, C::N_CHUNK, false, false);
            bool ok = true;
            for (int kc = 0; kc < k_chunks; ++kc) {
                const int s = kc % C::NS;
                if (!mbar_wait(&full[s], (kc / C::NS) & 1, ab, p.timeout_ns, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t xa = smem_u32(stage_x(s)), wa = smem_u32(stage_w(s));
#pragma unroll
                for (int kk = 0; kk < C::BKK / 16; ++kk) {
                    const uint64_t adesc = sdesc(xa + kk * 32, 16, 1024, SW128);
#pragma unroll
                    for (int n = 0; n < C::N_MMA; ++n) {
                        const uint64_t bdesc = sdesc(wa + n * C::N_CHUNK * 128 + kk * 32, 16, 1024, SW128);
                        umma_ss(tmem + n * C::N_CHUNK, adesc, bdesc, idesc, (kc | kk) != 0);
                    }
                }
                umma_commit(&empty[s]);
            }
            umma_commit(done);
            if (!ok) mbar_wait_drain(done, 0, p.timeout_ns);  // no MMA may be in flight at teardown
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int token = row0 + r;
        const bool valid = token < p.n_tok;
        const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
        const bool go = __all_sync(0xffffffffu, mbar_wait(done, 0, ab, p.timeout_ns, 3) && !ab->flag);
        if (go) {
            tc_fence_after();
            __nv_bfloat16* dst = nullptr;
            if (valid) {
                const int frame = token / p.T_f;
                const int slot = (p.first_slot + frame) % p.slots;
                const long long row = (long long)b * p.slots * p.T_f + (long long)slot * p.T_f + (token - frame * p.T_f);
                dst = p.cache + row * C::N;
            }
            float rstd = 1.0f;
            uint32_t v[32];
            if (p.normalize) {
                float ss = 0.f;
#pragma unroll 1
                for (int c = 0; c < DC; c += 32) {
                    tmem_ld_32x32b_x32(trow + c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float f = __uint_as_float(v[i]);
                        ss = fmaf(f, f, ss);
                    }
                }
                rstd = rsqrtf(ss * (1.0f / DC) + p.eps);
            }
#pragma unroll 1
            for (int c = 0; c < C::N; c += 32) {
                const int ncol = (C::N - c) < 32 ? 16 : 32;  // DR may leave a 16-column tail
                if (ncol == 32) {
                    tmem_ld_32x32b_x32(trow + c, v);
                } else {
                    uint32_t (&v16)[16] = *reinterpret_cast<uint32_t (*)[16]>(v);
                    tmem_ld_32x32b_x16(trow + c, v16);
                }
                tmem_wait_ld();
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float a = __uint_as_float(v[2 * i]), bb = __uint_as_float(v[2 * i + 1]);
                    const int col = c + 2 * i;
                    if (col < DC && p.normalize) {
                        const float g0 = p.gamma ? __ldg(p.gamma + col) : 1.f;
                        const float g1 = p.gamma ? __ldg(p.gamma + col + 1) : 1.f;
                        a = a * rstd * g0;
                        bb = bb * rstd * g1;
                    }
                    packed[i] = pack_bf16(a, bb);
                }
                if (valid) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c);
                    for (int q = 0; q < ncol / 8; ++q)
                        d4[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

}  // namespace vmla
