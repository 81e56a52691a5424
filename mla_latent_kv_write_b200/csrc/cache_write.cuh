// cache_write.cuh -- latent ring-cache write of "VideoMLA: Low-Rank Latent KV
// Cache for Minute-Scale Autoregressive Video Diffusion" (arXiv 2605.30351):
// [c | k^R] = x [W_dkv ; W_kr]^T (Sec. 3.1 Eq. 1, Sec. 3.2 Eq. 5), RMSNorm of
// the latent part (App. D.2), bf16 rows written into the FIFO frame ring
// (App. D.4).  k^R is stored unrotated and unnormalised.
//
// Two kernels, chosen by the number of 128-token tiles in the call:
//
// cache_write_cluster_kernel -- few tiles (a 4680-token chunk has 37, far fewer
// than the 148 SMs).  One thread-block cluster of ``ksplit`` CTAs (1 to 4) per
// tile; CTA r of the cluster accumulates the K range [r, r+1) * d_model / ksplit,
// so the tile's tensor-core and load work spreads over ksplit SMs.
// 192 threads per CTA:
//   warp 0     TMA producer (x tile 128 x 64 and W tile N x 64 per stage)
//   warp 1     tcgen05.mma issuer (M = 128, N = d_c + d_rope, K = 16 steps)
//              and tensor-memory owner
//   warps 2-5  epilogue.  After a cluster barrier (every CTA's MMAs are done,
//              so every CTA's pipeline stages are free) each thread copies one
//              TMEM lane (token row) of its fp32 partial into local shared
//              memory; each warp then ships its 32 rows to the peers that own
//              them (rows [128 r / ksplit, 128 (r+1) / ksplit) belong to rank r)
//              with bulk shared-to-shared copies completing on the peer's
//              mbarrier.
//   all warps  each owner sums the ksplit partials of its rows (a quad of
//              threads per row), reduces the row's sum of squares with warp
//              shuffles, applies RMSNorm and writes the row as 16-byte bf16 stores.
//
// cache_write_stream_kernel -- many tiles (batched chunks, long prefills).  A
// persistent grid of one CTA per SM walks the tiles; each tile's whole K range
// runs on one SM.  Warps 0 and 1 as above, with two tensor-memory accumulators
// when N <= 256, so that the next tile's MMAs overlap this tile's epilogue;
// warps 2-5 normalise their TMEM lanes (token rows) straight from tensor memory.
// It takes part in programmatic dependent launch: its prologue may run while the
// previous kernel of the stream finishes, and it waits for that kernel before it
// reads or writes global memory.
//
// Why a split of K across SMs stops at the cluster: every part holds the whole
// 128 x (d_c + d_rope) fp32 accumulator of the tile, so a split multiplies the
// epilogue's tensor-memory drain and its partial traffic by ksplit; through
// distributed shared memory inside a cluster that exchange is cheapest.
#pragma once

#include "ptx.cuh"

namespace vmla {

struct CacheWriteParams {
    int n_tok;            // tokens per batch element in this call
    int d_model;
    int ksplit;           // cluster kernel: CTAs per cluster along K (1 to 4)
    int tiles;            // stream kernel: 128-token tiles per batch element
    int units;            // stream kernel: batch * tiles
    int k_chunks;         // stream kernel: 64-wide K chunks per tile
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
struct ClusterWriteCfg {
    static constexpr int N = DC + DR;                 // cached scalars per token
    static constexpr int BM = 128;                    // tokens per tile
    static constexpr int BKK = 64;                    // K elements per stage (one 128-B swizzle row)
    static constexpr int N_MMA = N <= 256 ? 1 : 2;    // MMA column chunks
    static constexpr int N_CHUNK = N / N_MMA;
    // pipeline stages: as many as fit (the bytes in flight per SM set its streaming rate)
    static constexpr int NS = N <= 256 ? ((BM * BKK * 2 + N * BKK * 2) * 5 + 2048 + DC * 4 <= 232448 ? 5 : 4) : 3;
    static constexpr int X_BYTES = BM * BKK * 2;
    static constexpr int W_BYTES = N * BKK * 2;
    static constexpr int STAGE = X_BYTES + W_BYTES;
    static constexpr int WBOX = DC <= 192 ? DC : 192; // rows per W_dkv TMA box
    static constexpr int TMEM_COLS = N <= 256 ? 256 : 512;
    static constexpr int RED_STRIDE = N + 4;          // fp32 words per partial row (bank-conflict pad)
    static constexpr int PART_BYTES = BM * RED_STRIDE * 4;               // this CTA's fp32 partial
    static constexpr int SMEM_LIMIT = 232448;                            // opt-in shared memory per CTA
    // rows received from the peers for a K split ks: (ks - 1) * ceil(128 / ks)
    static constexpr int recv_rows(int ks) { return (ks - 1) * ((BM + ks - 1) / ks); }
    static constexpr bool fits(int ks) {
        return PART_BYTES + recv_rows(ks) * RED_STRIDE * 4 + 1024 + 256 + DC * 4 <= SMEM_LIMIT;
    }
    static constexpr int KS_MAX = N > 256 ? 1 : fits(4) ? 4 : fits(3) ? 3 : fits(2) ? 2 : 1;  // cluster size
    static constexpr int RED_BYTES = PART_BYTES + recv_rows(KS_MAX) * RED_STRIDE * 4;
    static constexpr int BUF = NS * STAGE > RED_BYTES ? NS * STAGE : RED_BYTES;
    static constexpr int SMEM = BUF + 1024 + 256 + DC * 4;  // stages | barriers | gamma
    static_assert(SMEM <= SMEM_LIMIT, "shared memory");
    static constexpr int THREADS = 192;
    static_assert(N % 16 == 0 && N_CHUNK % 16 == 0 && N_CHUNK <= 256, "MMA N");
    static_assert(DC % 32 == 0 && DR % 16 == 0 && DC % WBOX == 0, "widths");
    static_assert(N % 8 == 0 && N / 8 <= 64 && DC % 8 == 0, "a warp covers a row in 8-column groups");
};

// Rows [r_lo, r_hi) of this CTA's tile: sum the KS partials (this CTA's in
// ``part``, the peers' in the ``rbuf`` slots), RMSNorm of the latent columns with
// the gain ``gs``, bf16 rows into the ring slot of their frame.  Four threads per
// row (a quad of lanes); thread q of the quad holds the 8-column groups q, q + 4,
// ... so that each step of the quad covers 128 contiguous bytes; the row's sum of
// squares is reduced over the quad with warp shuffles.  KS is a template argument
// so that every partial of a group is loaded before any is summed.
template <int DC, int DR, int KS>
__device__ __forceinline__ void cw_cluster_finish_rows(const CacheWriteParams& p, const float* part, const float* rbuf,
                                               const float* gs, int rows_max, int r_lo, int r_hi, int row0, int b,
                                               bool store) {
    using C = ClusterWriteCfg<DC, DR>;
    constexpr int N = C::N, GROUPS = N / 8, GPT = (GROUPS + 3) / 4;
    const int q = threadIdx.x & 3;
    for (int r0 = r_lo; r0 < r_hi; r0 += C::THREADS / 4) {  // warp-uniform trip count
        const int r = r0 + int(threadIdx.x >> 2);
        const int token = row0 + r;
        const bool live = store && r < r_hi && token < p.n_tok;
        float a[GPT][8];
#pragma unroll
        for (int i = 0; i < GPT; ++i) {
            const int grp = q + 4 * i;
#pragma unroll
            for (int e = 0; e < 8; ++e) a[i][e] = 0.f;
            if (live && grp < GROUPS) {
                float4 u[KS][2];
#pragma unroll
                for (int k = 0; k < KS; ++k) {
                    const float* src = k == 0 ? part + r * C::RED_STRIDE + 8 * grp
                                              : rbuf + ((k - 1) * rows_max + (r - r_lo)) * C::RED_STRIDE + 8 * grp;
                    u[k][0] = *reinterpret_cast<const float4*>(src);
                    u[k][1] = *reinterpret_cast<const float4*>(src + 4);
                }
#pragma unroll
                for (int k = 0; k < KS; ++k) {
                    a[i][0] += u[k][0].x; a[i][1] += u[k][0].y; a[i][2] += u[k][0].z; a[i][3] += u[k][0].w;
                    a[i][4] += u[k][1].x; a[i][5] += u[k][1].y; a[i][6] += u[k][1].z; a[i][7] += u[k][1].w;
                }
            }
        }
        float scale = 1.0f;
        if (p.normalize) {
            float ss = 0.f;
#pragma unroll
            for (int i = 0; i < GPT; ++i)
                if (q + 4 * i < DC / 8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) ss = fmaf(a[i][e], a[i][e], ss);
                }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            scale = rsqrtf(ss * (1.0f / DC) + p.eps);
        }
        if (live) {
            const int frame = token / p.T_f;
            const int slot = (p.first_slot + frame) % p.slots;
            const long long row = (long long)b * p.slots * p.T_f + (long long)slot * p.T_f + (token - frame * p.T_f);
            uint4* out = reinterpret_cast<uint4*>(p.cache + row * N);
#pragma unroll
            for (int i = 0; i < GPT; ++i) {
                const int grp = q + 4 * i;
                if (grp < GROUPS) {
                    const bool norm = p.normalize && grp < DC / 8;
                    float o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = norm ? a[i][e] * scale * gs[8 * grp + e] : a[i][e];
                    out[grp] = make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                                          pack_bf16(o[6], o[7]));
                }
            }
        }
    }
}

template <int DC, int DR>
__global__ void __launch_bounds__(192, 1)
    cache_write_cluster_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wdkv,
                       const __grid_constant__ CUtensorMap tm_wkr, const CacheWriteParams p) {
    using C = ClusterWriteCfg<DC, DR>;
    constexpr int N = C::N;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BUF);
    uint64_t* empty = full + C::NS;
    uint64_t* done = empty + C::NS;
    uint64_t* recv = done + 1;  // partials of the peers for the rows this CTA owns
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv + 1);
    AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);
    float* part = reinterpret_cast<float*>(smem);  // fp32 partial [BM][RED_STRIDE], reuses the stages
    float* rbuf = reinterpret_cast<float*>(smem + C::PART_BYTES);  // [ks-1][rows_max][RED_STRIDE]
    float* gs = reinterpret_cast<float*>(smem + C::BUF + 256);      // RMSNorm gain [DC]

    const int warp = warp_id(), lane = lane_id();
    const int row0 = blockIdx.x * C::BM;
    const int b = blockIdx.z;
    const uint32_t rank = cluster_ctarank();
    const int k_chunks = p.d_model / C::BKK / p.ksplit;
    const int kc0 = int(rank) * k_chunks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(recv, 1);
        ab->flag = 0;
        if (p.ksplit > 1) {  // bytes the peers will send for this CTA's rows
            const int rows_mine = (C::BM * (int(rank) + 1)) / p.ksplit - (C::BM * int(rank)) / p.ksplit;
            mbar_arrive_expect_tx(recv, uint32_t((p.ksplit - 1) * rows_mine * C::RED_STRIDE * 4));
        }
        fence_mbar_init();
    }
    for (int c = threadIdx.x; c < DC; c += C::THREADS) gs[c] = p.gamma != nullptr ? __ldg(p.gamma + c) : 1.0f;
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
                const int kx = (kc0 + kc) * C::BKK;
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                tma_load_3d(stage_x(s), &tm_x, &full[s], kx, row0, b);
                for (int r = 0; r < DC; r += C::WBOX) tma_load_2d(stage_w(s) + r * 128, &tm_wdkv, &full[s], kx, r);
                tma_load_2d(stage_w(s) + DC * 128, &tm_wkr, &full[s], kx, 0);
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
    }

    // epilogue warps: the MMAs of this CTA are complete before the cluster barrier
    const int quarter = warp & 3;
    const uint32_t trow = tmem + (uint32_t(quarter * 32) << 16);
    bool go = true;
    if (warp >= 2) go = __all_sync(0xffffffffu, mbar_wait(done, 0, ab, p.timeout_ns, 3) && !ab->flag);

    // every thread of every CTA of the cluster takes this barrier: after it every
    // CTA's pipeline stages are free to receive partials
    tc_fence_before();
    cluster_sync();

    // abort flags of the peers (no peer can finish before it has received our rows)
    bool any_abort = false;
    for (int k = 0; k < p.ksplit; ++k)
        any_abort |= ld_dsmem_s32(mapa_shared(smem_u32(const_cast<int*>(&ab->flag)), uint32_t(k))) != 0;

    const int rows_max = (C::BM + p.ksplit - 1) / p.ksplit;
    if (warp >= 2) {
        // (a) TMEM lane (token row) r -> part[r][0 .. N), 128 columns per wait
        if (go) {
            tc_fence_after();
            const int r = quarter * 32 + lane;
            float* dst = part + r * C::RED_STRIDE;
#pragma unroll 1
            for (int c0 = 0; c0 < N; c0 += 128) {
                uint32_t v[4][32];
                const int nc = N - c0 < 128 ? N - c0 : 128;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (32 * q + 32 <= nc) tmem_ld_32x32b_x32(trow + c0 + 32 * q, v[q]);
                    else if (32 * q + 16 <= nc) tmem_ld_32x32b_x16(trow + c0 + 32 * q, *reinterpret_cast<uint32_t (*)[16]>(v[q]));
                }
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (32 * q + 4 * e + 4 <= nc)
                            *reinterpret_cast<float4*>(dst + c0 + 32 * q + 4 * e) =
                                make_float4(__uint_as_float(v[q][4 * e]), __uint_as_float(v[q][4 * e + 1]),
                                            __uint_as_float(v[q][4 * e + 2]), __uint_as_float(v[q][4 * e + 3]));
            }
        }
        fence_proxy_async_smem();  // the bulk copies read part through the async proxy
        __syncwarp();
        // (b) this warp's 32 rows go to the peers that own them as soon as they are
        // written (one bulk shared-to-shared copy per owner), overlapping the other
        // warps' TMEM reads; the copies complete on the owner's mbarrier
        if (lane == 0 && p.ksplit > 1) {
            for (int k = 0; k < p.ksplit; ++k) {
                if (k == int(rank)) continue;
                const int lo = (C::BM * k) / p.ksplit, hi = (C::BM * (k + 1)) / p.ksplit;
                const int a = max(quarter * 32, lo), e = min(quarter * 32 + 32, hi);
                if (a >= e) continue;
                const int slot = int(rank) < k ? int(rank) : int(rank) - 1;
                const uint32_t dst =
                    mapa_shared(smem_u32(rbuf + (slot * rows_max + (a - lo)) * C::RED_STRIDE), uint32_t(k));
                bulk_copy_to_peer(dst, smem_u32(part + a * C::RED_STRIDE), uint32_t((e - a) * C::RED_STRIDE * 4),
                                  mapa_shared(smem_u32(recv), uint32_t(k)));
            }
            bulk_commit();
        }
    }
    // every thread of the CTA: all of ``part`` is written before anyone reads its own rows
    __syncthreads();

    // (c) all 192 threads: sum the ksplit partials of this CTA's rows, RMSNorm, bf16 rows
    const bool got = p.ksplit == 1 || __all_sync(0xffffffffu, mbar_wait(recv, 0, ab, p.timeout_ns, 4));
    const int r_lo = (C::BM * int(rank)) / p.ksplit, r_hi = (C::BM * (int(rank) + 1)) / p.ksplit;
    const bool store = got && !any_abort && !ab->flag;
    switch (p.ksplit) {
        case 1: cw_cluster_finish_rows<DC, DR, 1>(p, part, rbuf, gs, rows_max, r_lo, r_hi, row0, b, store); break;
        case 2: cw_cluster_finish_rows<DC, DR, 2>(p, part, rbuf, gs, rows_max, r_lo, r_hi, row0, b, store); break;
        case 3: cw_cluster_finish_rows<DC, DR, 3>(p, part, rbuf, gs, rows_max, r_lo, r_hi, row0, b, store); break;
        default: cw_cluster_finish_rows<DC, DR, 4>(p, part, rbuf, gs, rows_max, r_lo, r_hi, row0, b, store); break;
    }
    // our outgoing copies must have read ``part`` before this CTA exits
    if (warp >= 2 && lane == 0 && p.ksplit > 1) bulk_wait_read();

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int DC, int DR>
struct StreamWriteCfg {
    static constexpr int N = DC + DR;                 // cached scalars per token
    static constexpr int BM = 128;                    // tokens per tile
    static constexpr int BKK = 64;                    // K elements per stage (one 128-B swizzle row)
    static constexpr int N_MMA = N <= 256 ? 1 : 2;    // MMA column chunks
    static constexpr int N_CHUNK = N / N_MMA;
    static constexpr int X_BYTES = BM * BKK * 2;
    static constexpr int W_BYTES = N * BKK * 2;
    static constexpr int STAGE = X_BYTES + W_BYTES;
    static constexpr int WBOX = DC <= 192 ? DC : 192; // rows per W_dkv TMA box
    static constexpr int NBUF = N <= 256 ? 2 : 1;     // tensor-memory accumulators
    static constexpr int TMEM_COLS = 512;
    static constexpr int SMEM_LIMIT = 232448;         // opt-in shared memory per CTA
    static constexpr int TAIL = DC * 4 + 256;         // gamma, barriers
    static constexpr int NS = (SMEM_LIMIT - 1024 - TAIL) / STAGE;  // pipeline stages
    static constexpr int SMEM = NS * STAGE + TAIL + 1024;
    static constexpr int THREADS = 192;
    static_assert(N % 16 == 0 && N_CHUNK % 16 == 0 && N_CHUNK <= 256, "MMA N");
    static_assert(DC % 32 == 0 && DR % 16 == 0 && DC % WBOX == 0, "widths");
    static_assert(STAGE % 1024 == 0 && NS >= 2 && NS <= 8, "stages");
};

// Load columns [c0, c0 + 32) (or 16 at the ragged end) of this warp's TMEM lanes.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, int c0, uint32_t (&v)[32]) {
    if (c0 + 32 <= N) tmem_ld_32x32b_x32(taddr + c0, v);
    else tmem_ld_32x32b_x16(taddr + c0, *reinterpret_cast<uint32_t(*)[16]>(v));
}

__device__ __forceinline__ long long cache_row(const CacheWriteParams& p, int b, int token) {
    const int frame = token / p.T_f;
    const int slot = (p.first_slot + frame) % p.slots;
    return (long long)b * p.slots * p.T_f + (long long)slot * p.T_f + (token - frame * p.T_f);
}

// ksplit == 1: thread = token row of this warp's lane quarter, straight from TMEM.
template <int DC, int DR>
__device__ __forceinline__ void cw_finish_tmem(const CacheWriteParams& p, uint32_t taddr, const float* gs, int b,
                                               int token, bool live) {
    using C = StreamWriteCfg<DC, DR>;
    constexpr int N = C::N;
    float ss = 0.f;
    if (p.normalize) {
#pragma unroll 1
        for (int c0 = 0; c0 < DC; c0 += 32) {
            uint32_t v[32];
            tmem_ld_cols<DC>(taddr, c0, v);
            tmem_wait_ld();
            const int nc = DC - c0 < 32 ? DC - c0 : 32;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (e < nc) ss = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), ss);
        }
    }
    const float scale = p.normalize ? rsqrtf(ss * (1.0f / DC) + p.eps) : 1.0f;
    uint4* out = reinterpret_cast<uint4*>(p.cache + (live ? cache_row(p, b, token) : 0) * N);
#pragma unroll 1
    for (int c0 = 0; c0 < N; c0 += 32) {
        uint32_t v[32];
        tmem_ld_cols<N>(taddr, c0, v);
        tmem_wait_ld();
        if (live) {
            const int ng = (N - c0 < 32 ? N - c0 : 32) / 8;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                if (g < ng) {
                    float o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int c = c0 + 8 * g + e;
                        const float a = __uint_as_float(v[8 * g + e]);
                        o[e] = (p.normalize && c < DC) ? a * scale * gs[c] : a;
                    }
                    out[(c0 >> 3) + g] = make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]),
                                                    pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
                }
            }
        }
    }
}

template <int DC, int DR>
__global__ void __launch_bounds__(192, 1)
    cache_write_stream_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wdkv,
                              const __grid_constant__ CUtensorMap tm_wkr, const CacheWriteParams p) {
    using C = StreamWriteCfg<DC, DR>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* gs = reinterpret_cast<float*>(smem + NS * C::STAGE);  // RMSNorm gain [DC]
    uint64_t* bars = reinterpret_cast<uint64_t*>(gs + DC);
    uint64_t* full = bars;                // [NS]
    uint64_t* empty = full + NS;          // [NS]
    uint64_t* acc_full = empty + NS;      // [NBUF]
    uint64_t* acc_empty = acc_full + 2;   // [NBUF]
    uint64_t* done = acc_empty + 2;       // all MMAs of the CTA complete (teardown)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    AbortState* ab = reinterpret_cast<AbortState*>(tmem_slot + 1);

    const int warp = warp_id(), lane = lane_id();
    const int G = gridDim.x;
    griddep_launch_dependents();  // a dependent launch may start its prologue; it waits for us to finish

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < C::NBUF; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(done, 1);
        ab->flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_wdkv);
        tma_prefetch_desc(&tm_wkr);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    griddep_wait();  // inputs and cache may belong to the previous kernel of the stream
    for (int c = threadIdx.x; c < DC; c += C::THREADS) gs[c] = p.gamma != nullptr ? __ldg(p.gamma + c) : 1.0f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto stage_x = [&](int s) { return smem + s * C::STAGE; };
    auto stage_w = [&](int s) { return smem + s * C::STAGE + C::X_BYTES; };

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < p.units && ok; u += G) {
                const int b = u / p.tiles, t = u - b * p.tiles;
                for (int kc = 0; kc < p.k_chunks; ++kc, ++it) {
                    const int s = it % NS;
                    if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1, ab, p.timeout_ns, 1)) {
                        ok = false;
                        break;
                    }
                    const int kx = kc * C::BKK;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_3d(stage_x(s), &tm_x, &full[s], kx, t * C::BM, b);
                    for (int r = 0; r < DC; r += C::WBOX) tma_load_2d(stage_w(s) + r * 128, &tm_wdkv, &full[s], kx, r);
                    tma_load_2d(stage_w(s) + DC * 128, &tm_wkr, &full[s], kx, 0);
                }
            }
            if (!ok || ab->flag) {  // let the copies still in flight land before the CTA exits
                for (int j = it - NS < 0 ? 0 : it - NS; j < it; ++j)
                    mbar_wait_drain(&full[j % NS], (j / NS) & 1, p.timeout_ns);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, C::N_CHUNK, false, false);
            bool ok = true;
            int it = 0, j = 0;
            for (int u = blockIdx.x; u < p.units && ok; u += G, ++j) {
                const int buf = j % C::NBUF;
                if (j >= C::NBUF && !mbar_wait(&acc_empty[buf], ((j / C::NBUF) - 1) & 1, ab, p.timeout_ns, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + uint32_t(buf * 256);
                for (int kc = 0; kc < p.k_chunks; ++kc, ++it) {
                    const int s = it % NS;
                    if (!mbar_wait(&full[s], (it / NS) & 1, ab, p.timeout_ns, 3)) {
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
                            umma_ss(acc + n * C::N_CHUNK, adesc, bdesc, idesc, (kc | kk) != 0);
                        }
                    }
                    umma_commit(&empty[s]);
                }
                if (ok) umma_commit(&acc_full[buf]);
            }
            umma_commit(done);
            mbar_wait_drain(done, 0, p.timeout_ns);  // no MMA may be in flight at teardown
        }
    } else {
        // epilogue warps 2-5: warp w normalises and stores TMEM lanes 32 (w % 4) ..
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;  // token row of the tile held by this thread
        int j = 0;
        for (int u = blockIdx.x; u < p.units; u += G, ++j) {
            const int b = u / p.tiles, t = u - b * p.tiles;
            const int buf = j % C::NBUF;
            const bool got = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (j / C::NBUF) & 1, ab, p.timeout_ns, 4));
            if (!got || ab->flag) break;  // warps leave independently: no barrier among them follows
            tc_fence_after();
            const uint32_t taddr = tmem + uint32_t(buf * 256) + (uint32_t(quarter * 32) << 16);
            const int token = t * C::BM + r;
            cw_finish_tmem<DC, DR>(p, taddr, gs, b, token, token < p.n_tok);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);  // the accumulator may take tile j + NBUF
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
