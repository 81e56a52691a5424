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
// A pre-pass (rope_window_kernel) forms the active window once per call: every
// valid cached k^R is rotated by its window-local position into an fp16
// workspace.  Then one CTA per (128-query tile, head, batch element), 352 threads:
//   warp 0     TMA producer: q_nope / W_uk (prologue), key tiles (128 keys:
//              latent from the cache, rotated rope key from the workspace) into
//              a 4-stage ring, W_uv (epilogue)
//   warp 1     tensor-memory owner; issues the q_abs, S = Q K^T and W_uv MMAs
//   warps 2-9  softmax, 16 query rows each: q_abs -> bf16 Q in TMEM, q^R
//              rotation, fp32 online softmax (row max / sum reduced across the
//              4 threads of a row with warp shuffles), P -> TMEM, O rescale,
//              normalisation, W_uv epilogue and the output stores
//   warp 10    issues the O += P C MMAs
// The two MMA streams come from two threads so that S_{j+1} and PV_j are
// queued to the tensor core independently: neither waits behind the other's
// dependency.  Two softmax warps per SM sub-partition let one warp's exp2 (MUFU)
// overlap the other's FMA / pack work.
// Tensor memory (512 columns, fp32 unless noted):
//   O [0, d_c)  S [d_c, d_c+128)  P (bf16 pairs) [+128, +64)
//   Q (bf16 pairs of q_abs, then fp16 pairs of the rotated q^R)
// Both contractions read their A operand from TMEM (Q for S = Q K^T, P for
// O += P C) and their B operand from the swizzled shared-memory key tile: the
// content part is K-major for S and MN-major for P C, so one copy serves both.
#pragma once

#include "ptx.cuh"

namespace vmla {

// max(a, b, c) in one instruction (three-operand form of max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

struct AttnParams {
    int Nq, H;
    int T_f, grid_w, slots, oldest;
    // valid key rows as up to three contiguous runs: runs 0 and 1 are physical
    // rows of the ring cache (two when the ring wraps), run 2 the rows of the
    // pinned sink frames (their own cache, rows [0, n_sink T_f))
    int seg_start[3], seg_len[3];
    int n_sink;                    // sink frames (local t = 0 .. n_sink-1; FIFO frames follow)
    int ws_rows;                   // rotated-key workspace rows per batch element: (slots + n_sink) T_f
    int n_kt;                      // key tiles of the whole window
    // split-KV: the key tiles of one (query tile, head, batch) unit are split over
    // n_split CTAs of tiles_per_split tiles; each writes its unnormalised O and
    // per-row (max, sum) to part_o / part_ml, and the last of them to arrive
    // (counters, zeroed by the window pre-pass) merges and finishes the unit
    int n_split, tiles_per_split, n_units;
    // head-packed tiles (never with split-KV): CTA x takes rows [128 x, 128 x + 128)
    // of the batch element's head-major (head, query) row order, so a tile may end
    // with the first queries of the next head.  Every head attends the same latent
    // keys, so only the prologue (W_uk,h) and the epilogue (W_uv,h) see the head.
    int packed;
    float* part_o;                 // [n_units * n_split, BM, d_c] fp32
    float* part_ml;                // [n_units * n_split, BM, 2] fp32: row max (raw score), row sum
    int* counters;                 // [n_units]
    int q_first;                   // logical window index of query 0
    int n_t, n_h;                  // rope pairs of the t and h axes (w takes the rest)
    float omega[32];               // rope frequency of each pair
    float scale_log2;              // log2(e) / sqrt(d_nope + d_rope)
    const __nv_bfloat16* q_rope;   // [B, Nq, H, DR]
    __nv_bfloat16* out;            // [B, Nq, H, DV]
    float* lse;                    // [B, Nq, H] or null
    uint64_t timeout_ns;
};

// TMA descriptors of one launch.  The key tensors get one map per valid run of
// rows whose row extent ends at the end of the run, so a ragged last tile reads
// zeros (never rows of slots outside the window).
struct AttnMaps {
    CUtensorMap cc[3];  // cache latent part, per run: (d_c + d_rope, run rows, B), box (64, BK, 1), 128B swizzle
    CUtensorMap kr[3];  // rotated rope keys (fp16), per run: (d_rope, run rows, B), box (d_rope, BK, 1)
    CUtensorMap qn;     // q_nope (d_nope, H, Nq, B), box (16, 1, BM, 1), 32B swizzle
    CUtensorMap wuk;    // W_uk (d_c, H * d_nope), box (64, d_nope), 128B swizzle
    CUtensorMap wuv;    // W_uv (d_c, H * d_v), box (64, d_v), 128B swizzle
};

template <int DC_, int DR_, int DN_, int DV_>
struct AttnCfg {
    static constexpr int DC = DC_, DR = DR_, DN = DN_, DV = DV_;
    static constexpr int W = DC + DR;  // cached scalars per token
    static constexpr int BM = 128;
    // Q (bf16 pairs) stays in tensor memory next to O, S and P when all four fit
    // in its 512 columns with 128-key tiles; otherwise Q moves to shared memory
    // (the score MMAs read both operands from there) and key tiles shrink to 64.
    static constexpr bool QS = DC + 128 + 64 + W / 2 > 512;
    static constexpr int BK = QS ? 64 : 128;
    static constexpr int C_ATOMS = (DC + 63) / 64;       // 64-column blocks (the last may be half used)
    static constexpr int C_ATOM = BK * 128;              // one 64-column block of the key tile
    static constexpr int R_ROWB = DR * 2;                // bytes of rotated k^R per key (fp16)
    static constexpr uint32_t R_SW = DR == 16 ? SW32 : DR == 32 ? SW64 : SW128;
    static constexpr int STAGE = C_ATOMS * C_ATOM + BK * R_ROWB;
    static constexpr int QN_CHUNKS = DN / 16;
    static constexpr int QN_BYTES = QN_CHUNKS * BM * 32;
    static constexpr int WUK_ATOM = DN * 128, WUK_BYTES = C_ATOMS * WUK_ATOM;
    static constexpr int WUV_ATOM = DV * 128, WUV_BYTES = C_ATOMS * WUV_ATOM;
    static constexpr int OLAT_ATOM = BM * 128;
    // Q region (QS only): q_nope and W_uk for the prologue, then Q (bf16 q_abs in
    // 64-column K-major blocks, fp16 rotated q^R after them), then O_lat
    static constexpr int Q_ATOM = BM * 128;
    static constexpr int QR_OFF = C_ATOMS * Q_ATOM;
    static constexpr int WUK_OFF = (QN_BYTES + 1023) / 1024 * 1024;
    static constexpr int QBYTES = QS ? QR_OFF + BM * R_ROWB : 0;
    static constexpr int NS = (4 * STAGE + QBYTES + 2048 <= 232448) ? 4
                            : (3 * STAGE + QBYTES + 2048 <= 232448) ? 3 : 2;  // key-tile ring stages
    // W_uv (epilogue) spreads over consecutive ring stages, APS 64-column blocks each
    static constexpr int APS = STAGE / WUV_ATOM;
    static constexpr int WUV_STAGES = (C_ATOMS + APS - 1) / APS;
    // MMAs of N = DC (q_abs, P C) run as NMMA column halves of NCH <= 256
    static constexpr int NMMA = DC > 256 ? 2 : 1;
    static constexpr int NCH = DC / NMMA;
    // With Q in shared memory only two ring stages fit, so each stage is filled and
    // freed in two halves: latent blocks [0, LO_ATOMS) ("lo") and the rest with the
    // rotated RoPE keys ("hi").  The two N halves of the PV MMA are their last
    // readers, so a stage's lo half refills while PV still reads its hi half, and
    // the next score MMAs start on the lo blocks before the hi half has landed.
    static constexpr bool HALVES = QS && NMMA == 2 && C_ATOMS % 2 == 0;
    static constexpr int LO_ATOMS = HALVES ? C_ATOMS / 2 : C_ATOMS;
    static constexpr int O_COL = 0, S_COL = DC, P_COL = DC + BK, Q_COL = DC + BK + BK / 2;
    // With Q in shared memory the score tile is double-buffered: S_j in columns
    // S_COL + (j mod 2) BK, and P_j (bf16 pairs) over the first BK / 2 columns of
    // its own S buffer, so the next tile's score MMAs need not wait for the
    // softmax; S_{j+2} is issued once PV_j has read P_j.
    static constexpr bool S2 = QS;
    static constexpr int TMEM_END = QS ? S_COL + 2 * BK : Q_COL + W / 2;
    // head-packed tiles: the second head's output goes to columns that are idle
    // once O / l has been staged (O itself, or P and Q when O is narrower)
    static constexpr int OUT2_COL = DC >= DV ? O_COL : P_COL;
    static constexpr int SMEM = NS * STAGE + QBYTES + 1024 + 1024;
    static constexpr int SM_WARPS_PER_HALF = 4;                 // softmax warps per 16-lane half
    static constexpr int SM_WARPS = 2 * SM_WARPS_PER_HALF;
    static constexpr int THREADS = 32 * (3 + SM_WARPS);
    static_assert(DC % 32 == 0 && NCH % 64 == 0 || NMMA == 1, "latent width");
    static_assert(DC % 32 == 0 && NCH <= 256, "latent width");
    static_assert(!HALVES || NCH / 64 == LO_ATOMS, "PV half n reads latent blocks [n LO_ATOMS, (n + 1) LO_ATOMS)");
    static_assert(DR == 16 || DR == 32 || DR == 64, "rope width");
    static_assert(DN % 16 == 0 && DV % 32 == 0 && DV <= 256, "head widths");
    static_assert(TMEM_END <= 512 && S_COL + DV <= 512, "tensor memory budget");
    static_assert(QS || (DC >= DV ? DV <= DC : P_COL + DV <= 512), "second head output region");
    static_assert(SMEM <= 232448 && APS >= 1, "shared memory budget");
    static_assert(QS ? (WUK_OFF + WUK_BYTES <= QBYTES && C_ATOMS * OLAT_ATOM <= QBYTES)
                     : (QN_BYTES <= STAGE && WUK_BYTES <= STAGE && WUV_STAGES == 1 && C_ATOMS * OLAT_ATOM <= STAGE),
                  "prologue / epilogue buffers reuse the Q region or pipeline stages");
};

struct AttnBarriers {
    uint64_t full[4], empty[4];
    uint64_t full_hi[4], empty_hi[4];  // the hi halves of the stages (HALVES only)
    uint64_t pv_buf[2];                // PV of a tile whose P sits in S buffer b (S2 only)
    uint64_t s_full2[2];               // S_j complete in buffer j % 2 (S2 only)
    uint64_t part_done, last_known;  // split-KV: partial stored by every softmax warp / arrival counted
    int last_flag, skip_epilogue;
    uint64_t q_full, qabs_done, q_ready, s_full, s_free, p_full, pv_done, olat_ready, out_full, drain, drain2;
    uint64_t qabs_mid, q2_full, wuv2_full, out2_full;  // head-packed tiles that hold two heads
    uint32_t tmem_base;
    AbortState ab;
};

// Key tile j -> (run, first row inside the run, valid rows).
template <int BK>
__device__ __forceinline__ void key_tile(const AttnParams& p, int j, int& run, int& row, int& valid) {
    const int t0 = (p.seg_len[0] + BK - 1) / BK;
    const int t1 = t0 + (p.seg_len[1] + BK - 1) / BK;
    run = j < t0 ? 0 : (j < t1 ? 1 : 2);
    row = (j - (run == 0 ? 0 : run == 1 ? t0 : t1)) * BK;
    valid = min(BK, p.seg_len[run] - row);
}

// Rotate the pair (x, y) by theta: (x cos - y sin, x sin + y cos), packed as
// fp16x2.  The RoPE part of the score contraction runs as its own fp16 x fp16
// MMAs, whose 11-bit significand keeps the rounding of the rotated vectors 8x
// below bf16 (values are O(10), far inside the fp16 range).
__device__ __forceinline__ uint32_t rotate_pair(uint32_t v_bf16x2, float theta) {
    float sn, cs;
    sincosf(theta, &sn, &cs);
    const float x = bf16_lo(v_bf16x2), y = bf16_hi(v_bf16x2);
    return pack_f16(x * cs - y * sn, x * sn + y * cs);
}

// Angle of rope pair ``pr`` at window-local position (t, hh, ww).
__device__ __forceinline__ float rope_theta(const AttnParams& p, int pr, int t, int hh, int ww) {
    const int pos = pr < p.n_t ? t : (pr < p.n_t + p.n_h ? hh : ww);
    return float(pos) * p.omega[pr];
}

// Forming the active window (App. D.5): rotate every valid cached k^R of the
// window by its window-local (t, h, w) position, once per call, into the fp16
// workspace [B, (slots + n_sink) T_f, DR]: ring row R at row R, sink row r at
// row slots T_f + r.  Local t: sink frame s -> s, ring frame j frames after the
// oldest valid one -> n_sink + j (App. D.4-D.5).  One thread per (batch, valid
// row, 4 pairs).
template <int DC, int DR>
__global__ void __launch_bounds__(256) rope_window_kernel(const __nv_bfloat16* __restrict__ cache,
                                                          const __nv_bfloat16* __restrict__ sink,
                                                          __half* __restrict__ krot, const AttnParams p, int B) {
    constexpr int W = DC + DR, CH = DR / 8;
    // Launched programmatically: nothing is read before the previous kernel has
    // finished.  Only then may the attention start: its prologue reads queries
    // that kernel (or an earlier one) may have written, and nothing of ours.
    griddep_wait();
    griddep_launch_dependents();
    if (p.n_split > 1) {  // arrival counters of the split-KV attention launched next
        for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < p.n_units;
             i += (long long)gridDim.x * blockDim.x)
            p.counters[i] = 0;
    }
    const int ring_valid = p.seg_len[0] + p.seg_len[1];
    const int rows_valid = ring_valid + p.seg_len[2];
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long long)B * rows_valid * CH) return;
    const int ch = int(gid % CH);
    const long long t2 = gid / CH;
    const int vr = int(t2 % rows_valid);
    const int b = int(t2 / rows_valid);
    int t, pp;
    const __nv_bfloat16* src;
    size_t dst;
    if (vr < ring_valid) {
        const int R = vr < p.seg_len[0] ? p.seg_start[0] + vr : p.seg_start[1] + (vr - p.seg_len[0]);
        const int slot = R / p.T_f;
        pp = R - slot * p.T_f;
        t = slot - p.oldest;
        if (t < 0) t += p.slots;
        t += p.n_sink;
        src = cache + (size_t(b) * p.slots * p.T_f + R) * W;
        dst = size_t(b) * p.ws_rows + R;
    } else {
        const int r = vr - ring_valid;
        t = r / p.T_f;
        pp = r - t * p.T_f;
        src = sink + (size_t(b) * p.n_sink * p.T_f + r) * W;
        dst = size_t(b) * p.ws_rows + size_t(p.slots) * p.T_f + r;
    }
    const int hh = pp / p.grid_w, ww = pp - (pp / p.grid_w) * p.grid_w;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + DC) + ch);
    uint4 o;
    o.x = rotate_pair(v.x, rope_theta(p, 4 * ch + 0, t, hh, ww));
    o.y = rotate_pair(v.y, rope_theta(p, 4 * ch + 1, t, hh, ww));
    o.z = rotate_pair(v.z, rope_theta(p, 4 * ch + 2, t, hh, ww));
    o.w = rotate_pair(v.w, rope_theta(p, 4 * ch + 3, t, hh, ww));
    reinterpret_cast<uint4*>(krot + dst * DR)[ch] = o;
}

// SPLIT: this launch shares the key tiles of a unit over p.n_split CTAs (the
// split-KV epilogue is compiled only into that instance).
template <class C, bool SPLIT>
__global__ void __launch_bounds__(352, 1) attention_kernel(const __grid_constant__ AttnMaps maps, const AttnParams p) {
    constexpr int DC = C::DC, DR = C::DR, DN = C::DN, DV = C::DV, BM = C::BM, BK = C::BK, NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* qreg = smem + NS * C::STAGE;  // Q region (QS only)
    AttnBarriers* bar = reinterpret_cast<AttnBarriers*>(qreg + C::QBYTES);
    AbortState* ab = &bar->ab;
    auto stage = [&](int s) { return smem + s * C::STAGE; };
    griddep_launch_dependents();  // every CTA of this grid is resident or done before a dependent starts

    const int warp = warp_id(), lane = lane_id();
    const int b = SPLIT ? int(blockIdx.z) / p.n_split : int(blockIdx.z);
    const int split = SPLIT ? int(blockIdx.z) % p.n_split : 0;
    // Rows r < n1 of the tile are queries i0 + r of head h; with head-packed tiles
    // rows r >= n1 are queries r - n1 of head h + 1 (a "mixed" tile).
    const bool packed = !SPLIT && !C::QS && p.packed != 0;
    int h, i0, n1;
    if (packed) {
        const int g0 = int(blockIdx.x) * BM;
        h = g0 / p.Nq;
        i0 = g0 - h * p.Nq;
        n1 = min(BM, p.Nq - i0);
    } else {
        h = blockIdx.y;
        i0 = int(blockIdx.x) * BM;
        n1 = BM;
    }
    const bool mixed = packed && n1 < BM && h + 1 < p.H;
    auto row_of = [&](int r, int& hr, int& ir) -> bool {  // (head, query) of tile row r; false: no row
        hr = r < n1 ? h : h + 1;
        ir = r < n1 ? i0 + r : r - n1;
        return hr < p.H && ir < p.Nq;
    };
    const int kt0 = SPLIT ? split * p.tiles_per_split : 0;                       // first key tile of this split
    const int nt = SPLIT ? min(p.n_kt, kt0 + p.tiles_per_split) - kt0 : p.n_kt;  // key tiles of this CTA (>= 1)
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bar->full[s], 1);
            mbar_init(&bar->empty[s], 1);
            mbar_init(&bar->full_hi[s], 1);
            mbar_init(&bar->empty_hi[s], 1);
        }
        mbar_init(&bar->q_full, 1);
        mbar_init(&bar->qabs_done, 1);
        mbar_init(&bar->q_ready, C::SM_WARPS);
        mbar_init(&bar->s_full, 1);
        mbar_init(&bar->s_free, C::SM_WARPS);
        mbar_init(&bar->pv_buf[0], 1);
        mbar_init(&bar->pv_buf[1], 1);
        mbar_init(&bar->s_full2[0], 1);
        mbar_init(&bar->s_full2[1], 1);
        mbar_init(&bar->p_full, C::SM_WARPS);
        mbar_init(&bar->pv_done, 1);
        mbar_init(&bar->olat_ready, C::SM_WARPS);
        mbar_init(&bar->out_full, 1);
        mbar_init(&bar->drain, 1);
        mbar_init(&bar->drain2, 1);
        mbar_init(&bar->part_done, C::SM_WARPS);
        mbar_init(&bar->last_known, 1);
        mbar_init(&bar->qabs_mid, 1);
        mbar_init(&bar->q2_full, 1);
        mbar_init(&bar->wuv2_full, 1);
        mbar_init(&bar->out2_full, 1);
        bar->last_flag = 0;
        bar->skip_epilogue = 0;
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
            uint8_t* qn_dst = C::QS ? qreg : stage(NS - 2);
            uint8_t* wuk_dst = C::QS ? qreg + C::WUK_OFF : stage(NS - 1);
            // q_nope rows of head hh starting at query i (rows past the head's last
            // query, or before its first, read zeros) and W_uk,hh
            auto load_q = [&](uint64_t* bq, int hh, int i) {
                mbar_arrive_expect_tx(bq, C::QN_BYTES + C::WUK_BYTES);
                for (int c = 0; c < C::QN_CHUNKS; ++c)
                    tma_load_4d(qn_dst + c * BM * 32, &maps.qn, bq, c * 16, hh, i, b);
                for (int a = 0; a < C::C_ATOMS; ++a)
                    tma_load_2d(wuk_dst + a * C::WUK_ATOM, &maps.wuk, bq, a * 64, hh * DN);
            };
            load_q(&bar->q_full, h, i0);
            // Launched programmatically after the RoPE pre-pass, which lets it start
            // only once every kernel before the pass has finished: the queries and
            // W_uk are complete; the window (and the split counters the pass
            // clears) are read only after the pass has finished too.
            griddep_wait();
            // mixed tile: once the first q_abs MMAs have read the buffers, the second
            // head's rows (tile rows n1..127, zeros above them) and W_uk,h+1 replace them
            bool ok = true, round2 = false, wuv2 = false;
            auto second_head = [&]() {
                if (!mixed || round2) return true;
                if (!mbar_wait(&bar->qabs_mid, 0, ab, to, 12)) return false;
                load_q(&bar->q2_full, h + 1, -n1);
                round2 = true;
                return true;
            };
            int issued = 0;
            bool qabs_seen = false;
            for (int j = 0; j < nt + C::WUV_STAGES; ++j) {
                const int s = j % NS;
                if (j >= NS) {
                    ok = mbar_wait(&bar->empty[s], ((j / NS) - 1) & 1, ab, to, 10);
                } else if (!C::QS && s >= NS - 2 && !qabs_seen) {  // stage still holds q_nope / W_uk
                    ok = second_head() && (qabs_seen = mbar_wait(&bar->qabs_done, 0, ab, to, 11));
                }
                if (!ok) break;
                if (j < nt) {
                    int run, row, valid;
                    key_tile<BK>(p, kt0 + j, run, row, valid);
                    uint64_t* fh = C::HALVES ? &bar->full_hi[s] : &bar->full[s];  // barrier of the hi half
                    mbar_arrive_expect_tx(&bar->full[s], C::HALVES ? C::LO_ATOMS * C::C_ATOM : C::STAGE);
                    for (int a = 0; a < C::LO_ATOMS; ++a)
                        tma_load_3d(stage(s) + a * C::C_ATOM, &maps.cc[run], &bar->full[s], a * 64, row, b);
                    if constexpr (C::HALVES) {
                        if (j >= NS) ok = mbar_wait(&bar->empty_hi[s], ((j / NS) - 1) & 1, ab, to, 14);
                        if (!ok) break;
                        mbar_arrive_expect_tx(fh, C::STAGE - C::LO_ATOMS * C::C_ATOM);
                    }
                    for (int a = C::LO_ATOMS; a < C::C_ATOMS; ++a)
                        tma_load_3d(stage(s) + a * C::C_ATOM, &maps.cc[run], fh, a * 64, row, b);
                    tma_load_3d(stage(s) + C::C_ATOMS * C::C_ATOM, &maps.kr[run], fh, 0, row, b);
                } else {  // W_uv blocks [a0, a1) of the epilogue
                    if constexpr (C::HALVES) {
                        if (j >= NS) ok = mbar_wait(&bar->empty_hi[s], ((j / NS) - 1) & 1, ab, to, 15);
                        if (!ok) break;
                    }
                    const int a0 = (j - nt) * C::APS;
                    const int a1 = a0 + C::APS < C::C_ATOMS ? a0 + C::APS : C::C_ATOMS;
                    mbar_arrive_expect_tx(&bar->full[s], (a1 - a0) * C::WUV_ATOM);
                    for (int a = a0; a < a1; ++a)
                        tma_load_2d(stage(s) + (a - a0) * C::WUV_ATOM, &maps.wuv, &bar->full[s], a * 64, h * DV);
                }
                issued = j + 1;
            }
            ok = ok && second_head();  // a window of fewer tiles never reached stage NS - 2
            if (ok && mixed) {
                // W_uv,h+1 into the stage of W_uv,h once the first epilogue MMAs are done
                ok = mbar_wait(&bar->out_full, 0, ab, to, 13);
                if (ok) {
                    mbar_arrive_expect_tx(&bar->wuv2_full, C::C_ATOMS * C::WUV_ATOM);
                    for (int a = 0; a < C::C_ATOMS; ++a)
                        tma_load_2d(stage(nt % NS) + a * C::WUV_ATOM, &maps.wuv, &bar->wuv2_full, a * 64,
                                    (h + 1) * DV);
                    wuv2 = true;
                }
            }
            if (ab->flag) {  // let this CTA's copies land before it exits
                mbar_wait_drain(&bar->q_full, 0, to);
                if (round2) mbar_wait_drain(&bar->q2_full, 0, to);
                if (wuv2) mbar_wait_drain(&bar->wuv2_full, 0, to);
                for (int j = issued > NS ? issued - NS : 0; j < issued; ++j) {
                    mbar_wait_drain(&bar->full[j % NS], (j / NS) & 1, to);
                    if (C::HALVES && j < nt) mbar_wait_drain(&bar->full_hi[j % NS], (j / NS) & 1, to);
                }
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
                constexpr uint32_t id_qabs = idesc_bf16_f32(128, C::NCH, false, true);
                const uint32_t sq = smem_u32(C::QS ? qreg : stage(NS - 2));
                const uint32_t sw = smem_u32(C::QS ? qreg + C::WUK_OFF : stage(NS - 1));
                auto qabs_mma = [&](bool acc) {
#pragma unroll
                    for (int k = 0; k < C::QN_CHUNKS; ++k)
#pragma unroll
                        for (int n = 0; n < C::NMMA; ++n)
                            umma_ss(tmem + C::O_COL + n * C::NCH, sdesc(sq + k * BM * 32, 16, 256, SW32),
                                    sdesc(sw + n * (C::NCH / 64) * C::WUK_ATOM + k * 2048, C::WUK_ATOM, 1024, SW128),
                                    id_qabs, acc || k > 0);
                };
                qabs_mma(false);
                if (mixed) {
                    // second head: its q_nope rows are zero where the first head's are not
                    // (and vice versa), so accumulating both products gives each row its own
                    // head's q_abs exactly
                    umma_commit(&bar->qabs_mid);
                    ok = mbar_wait(&bar->q2_full, 0, ab, to, 37);
                    if (ok) {
                        tc_fence_after();
                        qabs_mma(true);
                    }
                }
                if (ok) {
                    umma_commit(&bar->qabs_done);
                    ok = mbar_wait(&bar->q_ready, 0, ab, to, 31);
                }
            }
            constexpr uint32_t id_s = idesc_bf16_f32(128, BK, false, false);
            constexpr uint32_t id_s_rope = idesc_f16_f32(128, BK, false, false);
            for (int j = 0; ok && j < nt; ++j) {
                // S_j = Q . K_j^T : K = DC latent (bf16) + DR rotated rope (fp16) columns
                const int s = j % NS;
                ok = mbar_wait(&bar->full[s], (j / NS) & 1, ab, to, 32);
                if constexpr (C::S2) {  // S buffer j % 2 holds P_{j-2} until PV_{j-2} has read it
                    if (ok && j >= 2) ok = mbar_wait(&bar->pv_buf[j & 1], ((j - 2) >> 1) & 1, ab, to, 33);
                } else {
                    if (ok && j > 0) ok = mbar_wait(&bar->s_free, (j - 1) & 1, ab, to, 33);
                }
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(stage(s));
                const uint32_t s_col = C::S_COL + (C::S2 ? (j & 1) * BK : 0);
                if constexpr (C::QS) {
                    const uint32_t sq = smem_u32(qreg);
#pragma unroll
                    for (int k = 0; k < DC / 16; ++k) {
                        if (C::HALVES && k == C::LO_ATOMS * 4) {  // the hi half of the stage
                            if (!mbar_wait(&bar->full_hi[s], (j / NS) & 1, ab, to, 39)) break;
                            tc_fence_after();
                        }
                        umma_ss(tmem + s_col, sdesc(sq + (k / 4) * C::Q_ATOM + (k % 4) * 32, 16, 1024, SW128),
                                sdesc(st + (k / 4) * C::C_ATOM + (k % 4) * 32, 16, 1024, SW128), id_s, k > 0);
                    }
                    if (ab->flag) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int k = 0; k < DR / 16; ++k)
                        umma_ss(tmem + s_col, sdesc(sq + C::QR_OFF + k * 32, 16, 8 * C::R_ROWB, C::R_SW),
                                sdesc(st + C::C_ATOMS * C::C_ATOM + k * 32, 16, 8 * C::R_ROWB, C::R_SW), id_s_rope, 1);
                } else {
#pragma unroll
                    for (int k = 0; k < DC / 16; ++k)
                        umma_ts(tmem + C::S_COL, tmem + C::Q_COL + k * 8,
                                sdesc(st + (k / 4) * C::C_ATOM + (k % 4) * 32, 16, 1024, SW128), id_s, k > 0);
#pragma unroll
                    for (int k = 0; k < DR / 16; ++k)
                        umma_ts(tmem + C::S_COL, tmem + C::Q_COL + DC / 2 + k * 8,
                                sdesc(st + C::C_ATOMS * C::C_ATOM + k * 32, 16, 8 * C::R_ROWB, C::R_SW), id_s_rope, 1);
                }
                umma_commit(C::S2 ? &bar->s_full2[j & 1] : &bar->s_full);
            }
            if (ok) {
                // out [128 x DV] = O_lat [128 x DC] . W_uv,h^T  (all K-major SW128).  With Q in
                // tensor memory, O / l is split into two bf16 parts (hi in stage nt+1, lo in
                // stage nt+2) so that its rounding stays ~2^-16; with Q in shared memory the
                // single bf16 part lives in the Q region.  W_uv block a is in stage nt + a / APS.
                for (int w = 0; ok && w < C::WUV_STAGES; ++w)
                    ok = mbar_wait(&bar->full[(nt + w) % NS], ((nt + w) / NS) & 1, ab, to, 35);
                ok = ok && mbar_wait(&bar->olat_ready, 0, ab, to, 36);
                if (ok && !*reinterpret_cast<volatile int*>(&bar->skip_epilogue)) {
                    tc_fence_after();
                    constexpr uint32_t id_o = idesc_bf16_f32(128, DV, false, false);
                    const uint32_t ao = smem_u32(C::QS ? qreg : stage((nt + 1) % NS));
                    const uint32_t ao2 = smem_u32(stage((nt + 2) % NS));
                    auto out_mma = [&](uint32_t col) {
#pragma unroll
                        for (int k = 0; k < DC / 16; ++k) {
                            const int a = k / 4;
                            const uint32_t bw = smem_u32(stage((nt + a / C::APS) % NS)) + (a % C::APS) * C::WUV_ATOM;
                            const uint64_t bd = sdesc(bw + (k % 4) * 32, 16, 1024, SW128);
                            const uint32_t off = a * C::OLAT_ATOM + (k % 4) * 32;
                            umma_ss(tmem + col, sdesc(ao + off, 16, 1024, SW128), bd, id_o, k > 0);
                            if constexpr (!C::QS) umma_ss(tmem + col, sdesc(ao2 + off, 16, 1024, SW128), bd, id_o, 1);
                        }
                    };
                    out_mma(C::S_COL);
                    umma_commit(&bar->out_full);
                    if (mixed) {  // the second head's rows: O / l . W_uv,h+1^T into idle columns
                        ok = mbar_wait(&bar->wuv2_full, 0, ab, to, 38);
                        if (ok) {
                            tc_fence_after();
                            out_mma(C::OUT2_COL);
                            umma_commit(&bar->out2_full);
                        }
                    }
                }
            }
            if (!ok) {  // no MMA may still run when the tensor memory is released
                umma_commit(&bar->drain);
                mbar_wait_drain(&bar->drain, 0, to);
            }
        }
    } else if (warp == 2 + 2 * C::SM_WARPS_PER_HALF) {
        // ------------------------------------------------------------ PV issuer
        if (lane == 0) {
            constexpr uint32_t id_pv = idesc_bf16_f32(128, C::NCH, false, true);
            bool ok = true;
            for (int jj = 0; ok && jj < nt; ++jj) {
                const int sp = jj % NS;
                ok = mbar_wait(&bar->p_full, jj & 1, ab, to, 34);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(stage(sp));
                const uint32_t p_col = C::S2 ? C::S_COL + (jj & 1) * BK : C::P_COL;
#pragma unroll
                for (int n = 0; n < C::NMMA; ++n) {
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_ts(tmem + C::O_COL + n * C::NCH, tmem + p_col + k * 8,
                                sdesc(st + n * (C::NCH / 64) * C::C_ATOM + k * 2048, C::C_ATOM, 1024, SW128), id_pv,
                                (jj > 0 || k > 0));
                    if (C::HALVES) umma_commit(n == 0 ? &bar->empty[sp] : &bar->empty_hi[sp]);
                }
                if (!C::HALVES) umma_commit(&bar->empty[sp]);
                if (C::S2) umma_commit(&bar->pv_buf[jj & 1]);
                umma_commit(&bar->pv_done);
            }
            umma_commit(&bar->drain2);
            mbar_wait_drain(&bar->drain2, 0, to);
        }
    } else if (warp < 2 + 2 * C::SM_WARPS_PER_HALF) {
        // ------------------------------------------------------------ softmax / epilogue
        // warps 2-9.  A warp may only touch TMEM lanes 32 (warp % 4) .. + 31 (its
        // quadrant); warps 2-5 own lanes 0-15 of their quadrant, warps 6-9 lanes
        // 16-31, so every query row belongs to exactly one warp and the row max /
        // sum need no exchange between warps.
        const int w4 = warp & 3;
        const int half = (warp - 2) >> 2;
        const int quad = lane & 3;
        const uint32_t tq = tmem + (uint32_t(w4 * 32) << 16);    // quadrant base (32x32b shapes)
        const uint32_t tb = tq + (uint32_t(half * 16) << 16);    // this warp's 16 lanes (16xNb shapes)
        const float sl = p.scale_log2;

        // prologue: Q = [bf16(q_abs) | fp16(RoPE3D(q^R))], one row per thread, into
        // TMEM or (QS) into the Q region of shared memory in the swizzled K-major
        // layout the score MMAs read; the two warps of a quadrant take alternate
        // 32-column chunks of q_abs
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bar->qabs_done, 0, ab, to, 40) && !ab->flag);
        if (ok) {
            tc_fence_after();
            const int r = w4 * 32 + lane;
#pragma unroll 1
            for (int c = 32 * half; c < DC; c += 64) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tq + C::O_COL + c, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                if constexpr (C::QS) {
                    uint8_t* row_base = qreg + (c / 64) * C::Q_ATOM + r * 128;
                    const int kc0 = (c % 64) / 8;  // first 16-byte chunk of these 32 columns
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4*>(row_base + (((kc0 + i) ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                } else {
                    tmem_st_32x32b_x16(tq + C::Q_COL + c / 2, pk);
                }
            }
            if (half == 0) {
                int hr, i;
                const bool has_row = row_of(r, hr, i);
                uint32_t qr[DR / 2];
#pragma unroll
                for (int e = 0; e < DR / 2; ++e) qr[e] = 0u;
                if (has_row) {
                    const uint4* src = reinterpret_cast<const uint4*>(p.q_rope + ((size_t(b) * p.Nq + i) * p.H + hr) * DR);
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
                if constexpr (C::QS) {
                    // rows of R_ROWB bytes with the 16-byte chunk index XOR-ed by address
                    // bits [7, 7 + log2(R_ROWB / 16)): the 32B / 64B / 128B swizzles
                    uint8_t* row_base = qreg + C::QR_OFF + r * C::R_ROWB;
                    constexpr int NCH16 = C::R_ROWB / 16;
#pragma unroll
                    for (int e = 0; e < NCH16; ++e) {
                        const int sw = ((r * C::R_ROWB) >> 7) & (NCH16 - 1);
                        *reinterpret_cast<uint4*>(row_base + ((e ^ sw) << 4)) =
                            make_uint4(qr[4 * e], qr[4 * e + 1], qr[4 * e + 2], qr[4 * e + 3]);
                    }
                } else if constexpr (DR == 16) {
                    tmem_st_32x32b_x8(tq + C::Q_COL + DC / 2, qr);
                } else if constexpr (DR == 32) {
                    tmem_st_32x32b_x16(tq + C::Q_COL + DC / 2, qr);
                } else {
                    tmem_st_32x32b_x32(tq + C::Q_COL + DC / 2, qr);
                }
            }
            if constexpr (C::QS) fence_proxy_async_smem();  // generic stores -> MMA operand reads
            else tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->q_ready);
        }

        griddep_wait();  // the stores below may not overtake the RoPE pre-pass

        // main loop.  16x256b layout: this thread holds rows
        //   R0 = w4*32 + half*16 + lane/4 and R1 = R0 + 8, 32 columns of each
        //   (columns 8k + 2 quad + {0, 1} of each 64-column half of the tile).
        float m_used[2] = {0.f, 0.f}, l_part[2] = {0.f, 0.f};
        for (int j = 0; ok && j < nt; ++j) {
            ok = __all_sync(0xffffffffu, C::S2 ? mbar_wait(&bar->s_full2[j & 1], (j >> 1) & 1, ab, to, 41)
                                               : mbar_wait(&bar->s_full, j & 1, ab, to, 41));
            if (!ok) break;
            tc_fence_after();
            constexpr int NC = BK / 64;  // 64-column halves of the tile
            uint32_t sv[NC][32];
            const uint32_t s_col = C::S_COL + (C::S2 ? (j & 1) * BK : 0);
#pragma unroll
            for (int c = 0; c < NC; ++c) tmem_ld_16x256b_x8(tb + s_col + 64 * c, sv[c]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->s_free);

            int run, row, valid;
            key_tile<BK>(p, kt0 + j, run, row, valid);
            if (valid < BK) {  // ragged last tile of a run: mask the missing keys
#pragma unroll
                for (int c = 0; c < NC; ++c)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
#pragma unroll
                        for (int e = 0; e < 2; ++e)
                            if (64 * c + 8 * k + 2 * quad + e >= valid)
                                sv[c][4 * k + e] = sv[c][4 * k + 2 + e] = 0xff800000u;  // -inf
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < NC; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    mx[0] = fmax3(mx[0], __uint_as_float(sv[c][4 * k]), __uint_as_float(sv[c][4 * k + 1]));
                    mx[1] = fmax3(mx[1], __uint_as_float(sv[c][4 * k + 2]), __uint_as_float(sv[c][4 * k + 3]));
                }
#pragma unroll
            for (int k = 0; k < 2; ++k) {  // the 4 threads of a row hold its 128 columns
                mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 1));
                mx[k] = fmaxf(mx[k], __shfl_xor_sync(0xffffffffu, mx[k], 2));
            }
            bool waited = false;
            if (j == 0) {
                m_used[0] = mx[0];
                m_used[1] = mx[1];
            } else {
                // Rescale only when some row's max grew by more than 2^8 in probability
                // units; otherwise keep the stale max (exact, p <= 256 fits bf16 / fp32).
                const bool need = (mx[0] - m_used[0]) * sl > 8.0f || (mx[1] - m_used[1]) * sl > 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (j - 1) & 1, ab, to, 42));
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
                    for (int cc = 0; cc + 64 <= DC; cc += 64) {
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
                    if constexpr (DC % 64 != 0) {  // last 32 columns
                        uint32_t o[16];
                        tmem_ld_16x256b_x4(tb + C::O_COL + DC - 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            o[4 * k + 0] = __float_as_uint(__uint_as_float(o[4 * k + 0]) * f[0]);
                            o[4 * k + 1] = __float_as_uint(__uint_as_float(o[4 * k + 1]) * f[0]);
                            o[4 * k + 2] = __float_as_uint(__uint_as_float(o[4 * k + 2]) * f[1]);
                            o[4 * k + 3] = __float_as_uint(__uint_as_float(o[4 * k + 3]) * f[1]);
                        }
                        tmem_st_16x256b_x4(tb + C::O_COL + DC - 32, o);
                    }
                }
            }
            // P = exp2(s * sl - m * sl), packed bf16 pairs for the 16x128b store:
            // rep kk (4 columns) <- pair (8k + 2 quad, +1) of column half c, kk = 8c + k.
            // The affine step and the row sums run as paired fp32 ops (one issue
            // slot per two columns); the softmax warps are issue-bound.
            const float2 sl2 = make_float2(sl, sl);
            const float2 nm0 = make_float2(-m_used[0] * sl, -m_used[0] * sl);
            const float2 nm1 = make_float2(-m_used[1] * sl, -m_used[1] * sl);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
            uint32_t pa[2 * 8 * NC];
#pragma unroll
            for (int c = 0; c < NC; ++c)
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
            if (!C::S2 && j > 0 && !waited) {  // P_{j-1} must have been consumed before P_j overwrites it
                ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (j - 1) & 1, ab, to, 43));
                if (!ok) break;
                tc_fence_after();
            }
            // (S2: P_j goes over this tile's own scores, already in registers; PV_{j-2},
            // the last reader of that buffer, completed before S_j was issued)
            const uint32_t p_col = C::S2 ? s_col : C::P_COL;
            if constexpr (NC == 2) {
                tmem_st_16x128b_x16(tb + p_col, pa);
            } else {
                tmem_st_16x128b_x8(tb + p_col, pa);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->p_full);
        }

        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar->pv_done, (nt - 1) & 1, ab, to, 44) && !ab->flag);
        bool last = true;  // this CTA finishes the unit (always, without split-KV)
        const int r_top = w4 * 32 + half * 16 + (lane >> 2);
        const int r_bot = r_top + 8;
        float m_fin[2] = {m_used[0], m_used[1]}, l_fin[2] = {0.f, 0.f}, f_own[2] = {1.f, 1.f};
        constexpr int MAXS = 8;             // most splits of one unit
        float f_oth[MAXS][2];               // scale of split s's partial in the merged sum
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                l_fin[k] = l_part[k];
                l_fin[k] += __shfl_xor_sync(0xffffffffu, l_fin[k], 1);
                l_fin[k] += __shfl_xor_sync(0xffffffffu, l_fin[k], 2);
            }
        }
        const int unit = (b * p.H + h) * int(gridDim.x) + int(blockIdx.x);
        if (SPLIT && ok) {
            // (1) this split's unnormalised O and (max, sum) -> workspace
            const size_t slot = size_t(unit) * p.n_split + split;
            float* po = p.part_o + slot * (BM * DC);
#pragma unroll 1
            for (int c32 = 0; c32 < DC / 32; c32 += 2) {
                uint32_t o[32];
                const bool full = c32 + 2 <= DC / 32;
                if (full) {
                    tmem_ld_16x256b_x8(tb + C::O_COL + c32 * 32, o);
                } else {
                    tmem_ld_16x256b_x4(tb + C::O_COL + c32 * 32, *reinterpret_cast<uint32_t(*)[16]>(o));
                }
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (!full && k >= 4) break;
                    const int col = c32 * 32 + 8 * k + 2 * quad;
                    *reinterpret_cast<float2*>(po + r_top * DC + col) =
                        make_float2(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1]));
                    *reinterpret_cast<float2*>(po + r_bot * DC + col) =
                        make_float2(__uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3]));
                }
            }
            if (quad == 0) {
                *reinterpret_cast<float2*>(p.part_ml + (slot * BM + r_top) * 2) = make_float2(m_used[0], l_fin[0]);
                *reinterpret_cast<float2*>(p.part_ml + (slot * BM + r_bot) * 2) = make_float2(m_used[1], l_fin[1]);
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->part_done);
            // (2) once all 8 warps have stored, count this split; the last to arrive merges
            if (warp == 2) {
                const bool stored = __all_sync(0xffffffffu, mbar_wait(&bar->part_done, 0, ab, to, 46));
                if (lane == 0) {
                    const int prev = stored ? atomicAdd(&p.counters[unit], 1) : -1;
                    bar->last_flag = prev == p.n_split - 1;
                    mbar_arrive(&bar->last_known);
                }
                __syncwarp();
            }
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->last_known, 0, ab, to, 47) && !ab->flag);
            last = ok && *reinterpret_cast<volatile int*>(&bar->last_flag) != 0;
            if (last) {
                __threadfence();
                // merged row max and sum over the splits (each split's m is a raw score)
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const int r = k ? r_bot : r_top;
                    float mt = m_used[k];
                    for (int sp = 0; sp < p.n_split; ++sp)
                        if (sp != split)
                            mt = fmaxf(mt, __ldcg(p.part_ml + ((size_t(unit) * p.n_split + sp) * BM + r) * 2));
                    f_own[k] = ex2((m_used[k] - mt) * sl);
                    float lsum = l_fin[k] * f_own[k];
#pragma unroll
                    for (int sp = 0; sp < MAXS; ++sp) {
                        f_oth[sp][k] = 0.f;
                        if (sp < p.n_split && sp != split) {
                            const float2 ml = __ldcg(reinterpret_cast<const float2*>(
                                p.part_ml + ((size_t(unit) * p.n_split + sp) * BM + r) * 2));
                            f_oth[sp][k] = ex2((ml.x - mt) * sl);
                            lsum += ml.y * f_oth[sp][k];
                        }
                    }
                    m_fin[k] = mt;
                    l_fin[k] = lsum;
                }
            }
        }
        if (ok && last) {
            float inv[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) inv[k] = 1.0f / l_fin[k];
            // O_lat = O / l, K-major SW128: hi + lo bf16 parts in stages (nt+1) % NS and
            // (nt+2) % NS, or (QS) one bf16 part in the Q region; all are idle: every S and
            // PV MMA has completed.  With split-KV, O is this split's O scaled to the merged
            // max plus every other split's stored O, likewise scaled.
            uint8_t* ol = C::QS ? qreg : stage((nt + 1) % NS);
            uint8_t* ol2 = stage((nt + 2) % NS);
#pragma unroll 1
            for (int c32 = 0; c32 < DC / 32; c32 += 2) {  // 64 columns, or the last 32
                uint32_t o[32];
                const bool full = c32 + 2 <= DC / 32;
                if (full) {
                    tmem_ld_16x256b_x8(tb + C::O_COL + c32 * 32, o);
                } else {
                    tmem_ld_16x256b_x4(tb + C::O_COL + c32 * 32, *reinterpret_cast<uint32_t(*)[16]>(o));
                }
                tmem_wait_ld();
                float v[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    v[4 * k + 0] = __uint_as_float(o[4 * k + 0]) * f_own[0];
                    v[4 * k + 1] = __uint_as_float(o[4 * k + 1]) * f_own[0];
                    v[4 * k + 2] = __uint_as_float(o[4 * k + 2]) * f_own[1];
                    v[4 * k + 3] = __uint_as_float(o[4 * k + 3]) * f_own[1];
                }
                if constexpr (SPLIT) {
                    for (int sp = 0; sp < p.n_split; ++sp) {
                        if (sp == split) continue;
                        const float* ps = p.part_o + (size_t(unit) * p.n_split + sp) * (BM * DC);
                        float fa = 0.f, fb = 0.f;
#pragma unroll
                        for (int q = 0; q < MAXS; ++q)
                            if (q == sp) {
                                fa = f_oth[q][0];
                                fb = f_oth[q][1];
                            }
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            if (!full && k >= 4) break;
                            const int col = c32 * 32 + 8 * k + 2 * quad;
                            const float2 t = __ldcg(reinterpret_cast<const float2*>(ps + r_top * DC + col));
                            const float2 u = __ldcg(reinterpret_cast<const float2*>(ps + r_bot * DC + col));
                            v[4 * k + 0] = fmaf(t.x, fa, v[4 * k + 0]);
                            v[4 * k + 1] = fmaf(t.y, fa, v[4 * k + 1]);
                            v[4 * k + 2] = fmaf(u.x, fb, v[4 * k + 2]);
                            v[4 * k + 3] = fmaf(u.y, fb, v[4 * k + 3]);
                        }
                    }
                }
                const int cc = c32 / 2;
                const int off_top = cc * C::OLAT_ATOM + r_top * 128 + 4 * quad;
                const int off_bot = cc * C::OLAT_ATOM + r_bot * 128 + 4 * quad;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (!full && k >= 4) break;
                    uint32_t hi, lo;
                    split_bf16(v[4 * k] * inv[0], v[4 * k + 1] * inv[0], hi, lo);
                    const int ot = off_top + ((k ^ (r_top & 7)) << 4);
                    *reinterpret_cast<uint32_t*>(ol + ot) =
                        C::QS ? pack_bf16(v[4 * k] * inv[0], v[4 * k + 1] * inv[0]) : hi;
                    if constexpr (!C::QS) *reinterpret_cast<uint32_t*>(ol2 + ot) = lo;
                    split_bf16(v[4 * k + 2] * inv[1], v[4 * k + 3] * inv[1], hi, lo);
                    const int ob = off_bot + ((k ^ (r_bot & 7)) << 4);
                    *reinterpret_cast<uint32_t*>(ol + ob) =
                        C::QS ? pack_bf16(v[4 * k + 2] * inv[1], v[4 * k + 3] * inv[1]) : hi;
                    if constexpr (!C::QS) *reinterpret_cast<uint32_t*>(ol2 + ob) = lo;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->olat_ready);

            if (p.lse != nullptr && quad == 0) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    int hr, i;
                    if (row_of(r_top + 8 * k, hr, i))
                        p.lse[(size_t(b) * p.Nq + i) * p.H + hr] = (m_fin[k] * sl + __log2f(l_fin[k])) * 0.69314718055994531f;
                }
            }

            // out rows of this quadrant, one per thread; the two warps of a quadrant
            // take alternate 32-column chunks.  A mixed tile's second-head rows read
            // their own output columns.
            ok = __all_sync(0xffffffffu, mbar_wait(&bar->out_full, 0, ab, to, 45) && !ab->flag);
            if (ok) {
                tc_fence_after();
                const int r = w4 * 32 + lane;
                int hr, i;
                const bool has_row = row_of(r, hr, i);
                const bool second = mixed && r >= n1;
                __nv_bfloat16* dst = p.out + ((size_t(b) * p.Nq + i) * p.H + hr) * DV;
                for (int pass = 0; ok && pass < (mixed ? 2 : 1); ++pass) {
                    const bool mine = second == (pass == 1);
                    if (!__any_sync(0xffffffffu, mine)) continue;
                    if (pass == 1) {
                        ok = __all_sync(0xffffffffu, mbar_wait(&bar->out2_full, 0, ab, to, 48) && !ab->flag);
                        if (!ok) break;
                        tc_fence_after();
                    }
                    const uint32_t col = pass == 1 ? C::OUT2_COL : C::S_COL;
#pragma unroll 1
                    for (int c = 32 * half; c < DV; c += 64) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tq + col + c, v);
                        tmem_wait_ld();
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
                        if (mine && has_row) {
                            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                        }
                    }
                }
            }
        } else if (ok) {
            // not the last split of this unit: the last one writes its output
            if (lane == 0) {
                bar->skip_epilogue = 1;
                mbar_arrive(&bar->olat_ready);
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
