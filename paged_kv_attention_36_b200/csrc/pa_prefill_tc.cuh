// pa_prefill_tc.cuh -- multi-query (chunked prefill) attention over the paged
// KV cache on the tcgen05 tensor cores.
//
// Same contract as prefill_kernel (pa_prefill.cuh): sequence b's last q_len_b
// cached tokens are the query rows, row (token i, query head g*G + j) of kv
// head g attends to the tokens at or before position L_b - q_len_b + i.  A CTA
// owns 128 such rows (one M = 128 tile) of one (sequence, kv head) and walks
// the sequence's pages in blocks of BN tokens (BN / 16 pages):
//
//   S_j = Q K_j^T        tcgen05.mma, A = Q (shared memory), B = K_j (shared
//                        memory), fp32 accumulator in TMEM (NS buffers, so
//                        S_{j+1} is computed while S_j is in the softmax)
//   P_j = 2^(S_j*c - m)  softmax warpgroup: thread i owns row i (TMEM lane i),
//                        masks, keeps the running max m and sum l, writes P_j
//                        as bf16 over the first half of S_j's columns
//   O  += P_j V_j        tcgen05.mma, A = P_j (TMEM), B = V_j (shared memory,
//                        MN-major), fp32 accumulator in TMEM, one MMA per page
//
// The running max is raised lazily: O and l are rescaled only when a row's
// block maximum exceeds the max in use by more than 2^8 (P stays <= 256, well
// inside bf16 and fp32), so most blocks skip the TMEM round trip of O.
//
// CPS CTAs share an SM (TMEM columns and shared memory are sized for it),
// so one CTA's prologue and epilogue overlap another's main loop.
//
// Warps: 0 streams K and V pages (one 2-D tiled TMA copy per page and 64-wide
// panel) into a ring of KS blocks; 1 allocates TMEM and one of its threads
// issues every MMA; 2-5 (one per TMEM lane quarter) load Q, run the softmax
// and write the output.  Completion flows through mbarriers: TMA -> k_full
// -> MMA -> s_full -> softmax -> p_full (+ TMA -> v_full) -> MMA -> v_empty
// (which also tells the softmax that O holds block j's P V).
// K and V halves of a ring stage are refilled separately (k_empty once Q K^T
// has read it, v_empty once P V has), and K is loaded one block ahead of V,
// so each has a full softmax step more of lead than a shared stage would give.
// Parity waits are exact only if the barrier cannot complete again before
// the wait: every wait here is on a phase whose next completion needs an
// action the waiting thread takes later (a copy it has not issued, a P it
// has not written, an MMA it has not issued).  Reusing s_full to release the
// K ring breaks this when NS < KS (S_{j-KS+NS} can finish before K_j is
// loaded) and deadlocks until the bounded wait gives up.
//
// The staged layout of a block is [D/64 panels][BN tokens][128 bytes] with the
// 128-byte swizzle, for K and V alike: K is then the K-major B operand of
// Q K^T (8-token groups 1024 bytes apart) and V the MN-major B operand of
// P V (64-wide panels of head_dim BN*128 bytes apart).  Q has the same
// [D/64][128 rows][128 bytes] layout.  V rows past the context in the
// sequence's last page are zeroed in shared memory before P V reads them, so
// an unused slot's bits (NaN included) cannot reach the output through a zero
// probability.
#pragma once

#include "pa_prefill.cuh"
#include "pa_tcgen05.cuh"

namespace pa {

template <int D, int BN, int KS, int NS>
struct TcPrefillCfg {
    static constexpr int kBM = 128;                 // query rows of a CTA
    static constexpr int kPanels = D / 64;
    static constexpr int kPanelQ = kBM * 128;       // bytes of one 64-wide panel of Q
    static constexpr int kPanelKV = BN * 128;       // bytes of one 64-wide panel of a K or V block
    static constexpr int kQBytes = kPanels * kPanelQ;
    static constexpr int kKBytes = kPanels * kPanelKV;
    static constexpr int kStage = 2 * kKBytes;      // K block then V block
    static constexpr int kPages = BN / 16;          // pages per block
    static constexpr int kPageBytes = 16 * D * 2;   // one (block, kv head) tile
    static constexpr int kStageOff = kQBytes;
    static constexpr int kBarOff = kStageOff + KS * kStage;
    static constexpr int kNumBars = 1 + 4 * KS + 2 * NS + 1;
    static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // + TMEM slot, alignment slack
    static constexpr int kThreads = 6 * 32;
    static constexpr int kColsUsed = NS * BN + D;  // S buffers, then O
    static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
    static_assert(BN % 64 == 0 && BN <= 256, "block of whole 64-token halves");
    static_assert(kColsUsed <= 512, "TMEM columns");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kPanelKV % 1024 == 0 && kPanelQ % 1024 == 0, "swizzle atoms 1024-byte aligned");
};

// One CTA's 128-row tile.  PREFIX = false: rows of sequence b's query tokens
// against its own pages, causal (PrefillParams, bf16 output).  PREFIX = true:
// rows (member, query head) of a shared-prefix group against one key split
// of the group's shared pages, all visible (PrefixParams, fp32 partials).
template <bool PREFIX, int D, int G, int BN, int KS, int NS, class Params>
__device__ __forceinline__ void tc_attention_tile(const Params& p) {
    using Cfg = TcPrefillCfg<D, BN, KS, NS>;
    static_assert(Cfg::kBM % G == 0, "a tile holds whole tokens (members)");
    constexpr bool kKOnV = KS >= 4;  // release K ring slots with the V ones (deep rings)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* qs = smem;
    uint8_t* stages = smem + Cfg::kStageOff;
    uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
    uint64_t* k_full = q_full + 1;  // K and V halves of a stage fill and drain separately
    uint64_t* v_full = k_full + KS;
    uint64_t* k_empty = v_full + KS;
    uint64_t* v_empty = k_empty + KS;
    uint64_t* s_full = v_empty + KS;
    uint64_t* p_full = s_full + NS;
    uint64_t* drain = p_full + NS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    __shared__ int s_abort;
    volatile int* abort = &s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.y;

    // ---- this tile's rows and the key pages it attends ----
    int nrows, row0, nkeys;  // rows of the task, the tile's first row, keys staged (0 .. nkeys-1)
    const int32_t* bt;       // block-table entries of the staged pages
    int L = 0, q0 = 0, first_pos = 0, first = 0, P = 0, pg0 = 0;
    if constexpr (!PREFIX) {
        const int b = int(blockIdx.x) / p.tiles_per_seq;
        const int tile = int(blockIdx.x) - b * p.tiles_per_seq;
        if (b >= p.B) return;
        const bool report = tile == 0 && g == 0 && threadIdx.x == 0;
        L = __ldg(p.context_lens + b);
        const int64_t cap = int64_t(p.M) * 16;
        if (L < 0 || L > cap) {
            if (report) raise_error(PA_DEVERR_CONTEXT);
            L = L < 0 ? 0 : int32_t(cap);
        }
        q0 = __ldg(p.cu_q_lens + b);
        int32_t q_len = __ldg(p.cu_q_lens + b + 1) - q0;
        if (q_len < 0 || q_len > L) {  // queries must be cached tokens of the sequence
            if (report) raise_error(PA_DEVERR_CONTEXT);
            q_len = q_len < 0 ? 0 : L;
        }
        nrows = q_len * G;
        row0 = tile * Cfg::kBM;
        if (row0 >= nrows) return;  // whole CTA, before any barrier or TMEM use
        first_pos = L - q_len;      // position of query token 0
        const int last_row = (row0 + Cfg::kBM < nrows ? row0 + Cfg::kBM : nrows) - 1;
        nkeys = first_pos + last_row / G + 1;  // tokens 0 .. nkeys-1 are visible to some row
        bt = p.block_tables + int64_t(b) * p.M;
    } else {
        const int gi = int(blockIdx.x) / p.tiles_per_group;
        const int tile = int(blockIdx.x) - gi * p.tiles_per_group;
        if (gi >= p.num_groups) return;
        first = __ldg(p.group_offsets + gi);
        int last = __ldg(p.group_offsets + gi + 1);
        P = __ldg(p.group_prefix_pages + gi);
        const bool report = tile == 0 && g == 0 && blockIdx.z == 0 && threadIdx.x == 0;
        if (first < 0 || last > p.B || last < first || last - first > p.max_group_size || P > p.M) {
            if (report) raise_error(PA_DEVERR_PREFIX);
            first = first < 0 ? 0 : (first > p.B ? p.B : first);
            last = last < first ? first : (last > p.B ? p.B : last);
            if (last - first > p.max_group_size) last = first + p.max_group_size;
            if (P > p.M) P = p.M;
        }
        nrows = (last - first) * G;
        row0 = tile * Cfg::kBM;
        if (P <= 0 || row0 >= nrows) return;
        const int per = prefix_split_pages(P, gridDim.z);
        pg0 = int(blockIdx.z) * per;
        const int pg1 = pg0 + per < P ? pg0 + per : P;
        if (pg0 >= pg1) return;
        nkeys = (pg1 - pg0) * 16;  // shared pages are whole
        bt = p.block_tables + int64_t(first) * p.M + pg0;  // the group leader's table
    }
    const int pages = (nkeys + 15) / 16;
    const int nblk = (nkeys + BN - 1) / BN;

    // Loads in flight while the barriers and TMEM are set up: the page ids of
    // block 0 (producer lanes) and this thread's Q row (softmax warps).
    const int32_t blk_first = (warp == 0 && lane < Cfg::kPages && lane < pages) ? __ldg(bt + lane) : 0;
    uint4 qv[D / 8];
    if (warp >= 2) {
        const int r = row0 + (warp & 3) * 32 + lane;
        const bool valid = r < nrows;
        const int64_t qrow = int64_t(PREFIX ? first : q0) + r / G;
        const int64_t orow = valid ? (qrow * p.Hq + g * G + r % G) * D : 0;
        const uint4* src = reinterpret_cast<const uint4*>(p.q + orow * 2);
#pragma unroll
        for (int ch = 0; ch < D / 8; ++ch) qv[ch] = valid ? __ldg(src + ch) : make_uint4(0u, 0u, 0u, 0u);
    }

    if (threadIdx.x == 0) {
        mbar_init(q_full, 128);
        for (int s = 0; s < KS; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int i = 0; i < NS; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 128);
        }
        mbar_init(drain, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_o = tmem + NS * BN;  // O columns; S buffer i at tmem + i*BN

    if (warp == 0) {
        // ======================= producer warp =======================
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_v)) : "memory");
        }
        const uint64_t pol = policy_evict_normal();  // the sequence's other row tiles read these pages too
        // K of block j, or V: its stage half is free once the MMA that read
        // it (Q K^T, or P V) has completed
        auto load = [&](int j, bool v, int32_t blk) -> bool {
            const int s = j % KS;
            uint64_t* full = v ? &v_full[s] : &k_full[s];
            // with a deep ring the K half is released with the V half (on
            // v_empty: its next completion needs V_j, loaded after K_j), which
            // saves the MMA thread a commit per block
            if (j >= KS && !__all_sync(0xffffffffu, mbar_wait_sleep((v || kKOnV) ? &v_empty[s] : &k_empty[s],
                                                                    uint32_t(j / KS - 1) & 1, abort)))
                return false;
            const int npg = pages - j * Cfg::kPages < Cfg::kPages ? pages - j * Cfg::kPages : Cfg::kPages;
            if (lane == 0) mbar_arrive_expect_tx(full, uint32_t(npg * Cfg::kPageBytes));
            __syncwarp();
            if (lane < npg) {
                if (blk < 0 || blk >= p.NB) {
                    raise_error(PA_DEVERR_BLOCK_ID);
                    blk = 0;
                }
                const int t = blk * p.Hkv + g;
                uint8_t* dst = stages + s * Cfg::kStage + (v ? Cfg::kKBytes : 0) + lane * 2048;
#pragma unroll
                for (int c = 0; c < Cfg::kPanels; ++c)
                    tma_load_4d(dst + c * Cfg::kPanelKV, v ? &p.tmap_v : &p.tmap_k, 0, 0, c, t, full, pol);
            }
            return true;
        };
        // lane i's page of block t (read one block ahead, so the table load
        // overlaps the waits)
        auto page_of = [&](int t) -> int32_t {
            const int pg = t * Cfg::kPages + lane;
            return (t < nblk && lane < Cfg::kPages && pg < pages) ? __ldg(bt + pg) : 0;
        };
        // K runs one block ahead of V: V_j is read one softmax step after K_j
        int nk = 0, nv = 0;  // blocks whose K (V) copies were issued
        int32_t blk_cur = blk_first, blk_prev = 0;
        for (int t = 0; t <= nblk; ++t) {
            const int32_t blk_next = page_of(t + 1);
            if (t < nblk) {
                if (!load(t, false, blk_cur)) break;
                nk = t + 1;
            }
            if (t >= 1) {
                if (!load(t - 1, true, blk_prev)) break;
                nv = t;
            }
            blk_prev = blk_cur;
            blk_cur = blk_next;
        }
        // every copy issued lands before shared memory is released
        if (lane == 0) {
            for (int i = (nk > KS ? nk - KS : 0); i < nk; ++i)
                mbar_wait_sleep(&k_full[i % KS], uint32_t(i / KS) & 1, nullptr, 20000000ull);
            for (int i = (nv > KS ? nv - KS : 0); i < nv; ++i)
                mbar_wait_sleep(&v_full[i % KS], uint32_t(i / KS) & 1, nullptr, 20000000ull);
        }
    } else if (warp == 1) {
        // ===================== MMA issue (one thread) =====================
        if (lane == 0) {
            constexpr uint32_t id_qk = idesc_bf16_f32(128, BN, false);
            constexpr uint32_t id_pv = idesc_bf16_f32(128, D, true);
            const uint64_t qd = sw128_desc(smem_u32(qs), 16, 1024);
            const uint32_t st0 = smem_u32(stages);
            bool ok = mbar_wait_sleep(q_full, 0, abort);
            // S_i = Q K_i^T into buffer i % NS, once the P V that last read
            // that buffer (block i - NS) has completed
            auto issue_qk = [&](int i) -> bool {
                const int s = i % KS, bb = i % NS;
                if (!mbar_wait_sleep(&k_full[s], uint32_t(i / KS) & 1, abort)) return false;
                if (i >= NS && !mbar_wait_sleep(&v_empty[(i - NS) % KS], uint32_t((i - NS) / KS) & 1, abort))
                    return false;
                tc_fence_after();
                // descriptors advance by (byte offset >> 4) in their address field
                const uint64_t kd = sw128_desc(st0 + s * Cfg::kStage, 16, 1024);
#pragma unroll
                for (int c = 0; c < Cfg::kPanels; ++c)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_ss(tmem + bb * BN, qd + uint64_t((c * Cfg::kPanelQ + kk * 32) >> 4),
                                kd + uint64_t((c * Cfg::kPanelKV + kk * 32) >> 4), id_qk, uint32_t(c | kk));
                umma_commit(&s_full[bb]);
                if (!kKOnV) umma_commit(&k_empty[s]);
                return true;
            };
            // S runs NS - 1 blocks ahead of P V.  Each step first issues the
            // next S (S_{j+NS-1} with three or more buffers, into the buffer
            // P_{j-1} V releases; S_{j+1} with two, after P_{j-1} V), then
            // waits for P_j and issues P_j V, so an S never waits behind the
            // softmax of the block before it.
            for (int i = 0; ok && i < NS - 1 && i < nblk; ++i) ok = issue_qk(i);
            for (int j = 0; ok && j < nblk; ++j) {
                if (j + NS - 1 < nblk && !(ok = issue_qk(j + NS - 1))) break;
                const int s = j % KS, bb = j % NS;
                ok = mbar_wait_sleep(&p_full[bb], uint32_t(j / NS) & 1, abort) &&
                     mbar_wait_sleep(&v_full[s], uint32_t(j / KS) & 1, abort);
                if (!ok) break;
                tc_fence_after();
                const int npg = pages - j * Cfg::kPages < Cfg::kPages ? pages - j * Cfg::kPages : Cfg::kPages;
                const uint64_t vd = sw128_desc(st0 + s * Cfg::kStage + Cfg::kKBytes, Cfg::kPanelKV, 1024);
                const uint32_t pa = tmem + bb * BN;
#pragma unroll
                for (int pg = 0; pg < Cfg::kPages; ++pg)
                    if (pg < npg) umma_ts(t_o, pa + pg * 8, vd + uint64_t(pg * (2048 >> 4)), id_pv, uint32_t(j | pg));
                umma_commit(&v_empty[s]);
            }
            // no MMA may still run when TMEM and shared memory are released
            umma_commit(drain);
            mbar_wait_sleep(drain, 0, nullptr, 20000000ull);
        }
        __syncwarp();
    } else {
        // ========================= softmax warpgroup =========================
        const int qw = warp & 3;                // TMEM lane quarter of this warp
        const int row = qw * 32 + lane;         // this thread's row of the tile
        const int gt = (warp - 2) * 32 + lane;  // 0..127 within the warpgroup
        const uint32_t lanes = uint32_t(qw * 32) << 16;
        const int r = row0 + row;
        const bool valid = r < nrows;
        // keys 0 .. lim-1 are visible to this row; its query row
        const int lim = PREFIX ? nkeys : (valid ? first_pos + r / G + 1 : 1);
        const int64_t qrow = int64_t(PREFIX ? first : q0) + r / G;

        // Q row into shared memory (128-byte swizzle: 16-byte chunk c of row t at c ^ (t % 8))
        {
#pragma unroll
            for (int ch = 0; ch < D / 8; ++ch)
                *reinterpret_cast<uint4*>(qs + (ch >> 3) * Cfg::kPanelQ + row * 128 + (((ch & 7) ^ (row & 7)) << 4)) =
                    qv[ch];
            fence_proxy_async_smem();
            mbar_arrive(q_full);
        }

        // the sequence's last page, when it is staged and ends inside the context
        const int rem = L & 15;
        const int last_pg = (L - 1) >> 4;
        const int zero_blk = (!PREFIX && rem != 0 && last_pg < pages) ? last_pg / Cfg::kPages : -1;

        const float c = p.qscale;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nblk; ++j) {
            const int bb = j % NS;
            ok = __all_sync(0xffffffffu, mbar_wait_sleep(&s_full[bb], uint32_t(j / NS) & 1, abort));
            if (!ok) break;
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int k = 0; k < BN / 64; ++k) tmem_ld64(tmem + lanes + bb * BN + 64 * k, &s[64 * k]);
            // logits in log2 units are s * ce: with a positive scale the scale
            // is applied inside the exponent's fma (the max commutes with it);
            // otherwise s is scaled first and ce = 1.  Keys past the row's
            // position -> -inf.
            const int n0 = j * BN;
            float ce = c;
            if (!(c > 0.f)) {
#pragma unroll
                for (int i = 0; i < BN; ++i) s[i] *= c;
                ce = 1.f;
            }
            if (n0 + BN > lim) {
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (n0 + i >= lim) s[i] = -INFINITY;
            }
            // row max over 8 independent partials (no BN-long dependency
            // chain), two logits per three-input max
            float mp[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mp[u] = s[u];
#pragma unroll
            for (int i = 8; i < BN; i += 2) mp[(i >> 1) & 7] = fmax3(mp[(i >> 1) & 7], s[i], s[i + 1]);
            const float m_blk =
                fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])) * ce;
            const float m_new = fmaxf(m, m_blk);
            if (__any_sync(0xffffffffu, m_new > m + 8.f)) {
                const float alpha = ex2_approx(m - m_new);  // 0 while m = -inf
                if (j > 0) {
                    ok = __all_sync(0xffffffffu,
                                    mbar_wait_sleep(&v_empty[(j - 1) % KS], uint32_t((j - 1) / KS) & 1, abort));
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < D / 32; ++k) {
                        float o[32];
                        tmem_ld32(t_o + lanes + 32 * k, o);
                        uint32_t w[32];
#pragma unroll
                        for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(o[i] * alpha);
                        tmem_st32(t_o + lanes + 32 * k, w);
                    }
                }
                l *= alpha;
                m = m_new;
            }
            // P = 2^(s*ce - m) as bf16 pairs over the first BN/2 columns of the
            // buffer; the exponent and the row sum in packed f32x2 arithmetic
            const uint64_t ce2 = f2_pack(ce, ce), nm2 = f2_pack(-m, -m);
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int k = 0; k < BN / 64; ++k) {
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float t0, t1;
                    f2_unpack(f2_fma(f2_pack(s[64 * k + 2 * i], s[64 * k + 2 * i + 1]), ce2, nm2), t0, t1);
                    const float p0 = ex2_approx(t0), p1 = ex2_approx(t1);
                    acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
                    w[i] = float2_to_bf16x2(p0, p1);
                }
                tmem_st32(tmem + lanes + bb * BN + 32 * k, w);
            }
            {
                float a0, a1, b0, b1;
                f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
                f2_unpack(f2_add(acc[2], acc[3]), b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            tmem_st_wait();
            if (j == zero_blk) {
                // V rows rem .. 15 of the last page hold no token of the context
                ok = __all_sync(0xffffffffu, mbar_wait_sleep(&v_full[j % KS], uint32_t(j / KS) & 1, abort));
                if (!ok) break;
                uint8_t* vz = stages + (j % KS) * Cfg::kStage + Cfg::kKBytes + (last_pg % Cfg::kPages) * 2048;
                const int pieces = (16 - rem) * 8;  // 16-byte pieces per panel
                for (int i = gt; i < pieces * Cfg::kPanels; i += 128) {
                    const int pc = i / pieces, rr = i - pc * pieces;
                    *reinterpret_cast<uint4*>(vz + pc * Cfg::kPanelKV + (rem + (rr >> 3)) * 128 + ((rr & 7) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            mbar_arrive(&p_full[bb]);
        }

        // ---- output: O / l (bf16 rows, or the split's fp32 partial rows).
        // Each thread writes its row into the Q and ring space, idle once the
        // last P V has completed (rows padded by 16 bytes, so a warp's 16-byte
        // writes fall in distinct banks); then every warp copies whole rows
        // out with consecutive lanes on consecutive 16 bytes.
        if (ok)
            ok = __all_sync(0xffffffffu,
                            mbar_wait_sleep(&v_empty[(nblk - 1) % KS], uint32_t((nblk - 1) / KS) & 1, abort));
        constexpr int kRowBytes = D * (PREFIX ? 4 : 2);
        constexpr int kRowStride = kRowBytes + 16;
        static_assert(Cfg::kBM * kRowStride <= Cfg::kBarOff, "output staging fits in the Q and ring space");
        if (ok) {
            tc_fence_after();
            const float inv = 1.f / l;
            uint8_t* mine = smem + row * kRowStride;
#pragma unroll
            for (int k = 0; k < D / 64; ++k) {
                float o[64];
                tmem_ld64(t_o + lanes + 64 * k, o);
                if constexpr (!PREFIX) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4*>(mine + (64 * k + 8 * q) * 2) =
                            make_uint4(float2_to_bf16x2(o[8 * q] * inv, o[8 * q + 1] * inv),
                                       float2_to_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv),
                                       float2_to_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv),
                                       float2_to_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv));
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        *reinterpret_cast<float4*>(mine + (64 * k + 4 * q) * 4) =
                            make_float4(o[4 * q] * inv, o[4 * q + 1] * inv, o[4 * q + 2] * inv, o[4 * q + 3] * inv);
                }
            }
            if constexpr (PREFIX) {
                // (max logit in base 2, exp-sum) of the row's partial
                if (valid) p.prefix_ml[(int64_t(blockIdx.z) * p.B + qrow) * p.Hq + g * G + r % G] = make_float2(m, l);
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the 4 softmax warps: rows staged
        if (!*abort) {
            constexpr int kChunks = kRowBytes / 16;       // 16-byte chunks per row
            constexpr int kRowsPerPass = 32 / kChunks;    // rows per warp instruction
            const int wq = warp - 2;
            for (int rr = wq * kRowsPerPass + lane / kChunks; rr < Cfg::kBM; rr += 4 * kRowsPerPass) {
                const int rg = row0 + rr;
                if (rg >= nrows) break;  // rows only grow along the loop
                const int ch = lane % kChunks;
                const uint4 v = *reinterpret_cast<const uint4*>(smem + rr * kRowStride + ch * 16);
                const int64_t qr = int64_t(PREFIX ? first : q0) + rg / G;
                const int64_t grow = (PREFIX ? int64_t(blockIdx.z) * p.B * p.Hq : int64_t(0)) + qr * p.Hq +
                                     g * G + rg % G;
                if constexpr (PREFIX)
                    reinterpret_cast<uint4*>(p.prefix_o + grow * D)[ch] = v;
                else
                    reinterpret_cast<uint4*>(p.out + grow * D)[ch] = v;
            }
        }
        if constexpr (PREFIX) {
            // checks of the caller's grouping: each member of the tile holds
            // the split's prefix blocks in its own table and its context covers
            // the whole prefix.  The (member, page) pairs are dealt out over the
            // Hkv CTAs of the tile and split (kv head g takes every Hkv-th run
            // of 128), so no CTA carries them all at its end.
            const int npg = nkeys / 16;
            const int m_lo = row0 / G;
            const int m_hi = ((row0 + Cfg::kBM < nrows ? row0 + Cfg::kBM : nrows) + G - 1) / G;
            for (int x = g * 128 + gt; x < (m_hi - m_lo) * npg; x += 128 * p.Hkv) {
                const int mem = first + m_lo + x / npg;
                const int j = pg0 + x % npg;
                if (__ldg(p.block_tables + int64_t(mem) * p.M + j) != __ldg(bt + (j - pg0)))
                    raise_error(PA_DEVERR_PREFIX);
                if (x % npg == 0 && int64_t(__ldg(p.context_lens + mem)) < int64_t(P) * 16)
                    raise_error(PA_DEVERR_PREFIX);
            }
        }
    }

    // ---- release TMEM once every warp's tcgen05 work has finished ----
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

template <int D, int G, int BN, int KS, int CPS, int NS>
__global__ void __launch_bounds__(6 * 32, CPS) prefill_tc_kernel(const __grid_constant__ PrefillParams p) {
    tc_attention_tile<false, D, G, BN, KS, NS>(p);
}

// The shared-prefix (cascade) pass on tcgen05: grid (group x row tile, kv
// head, key split); each CTA also copies its slice of the step's append.
template <int D, int G, int BN, int KS, int CPS, int NS>
__global__ void __launch_bounds__(6 * 32, CPS) prefix_tc_kernel(const __grid_constant__ PrefixParams p) {
    // the decode launched after this kernel may start its set-up now; it
    // waits for this grid to complete before it reads anything written here
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    prefix_append_slice<D>(p, 6 * 32);
    tc_attention_tile<true, D, G, BN, KS, NS>(p);
}

}  // namespace pa
