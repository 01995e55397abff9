// k_decode_mla.cu -- exact attention over the selected pages for the MLA geometry, on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Vortex paper note, section 系统设计 3: besides reusing dense attention backends the
// system adds its own kernel for more general MLA geometry; the MLA experiment section
// runs GLM-4.7-Flash (one shared latent KV per token: 512 latent + 64 rope dims; the
// first 512 dims are also the value).
//
// Geometry: 1 KV head, up to 16 query heads, Dqk = 576, Dv = 512, pages of 32 or 64
// tokens.  A tile is one selected page, loaded by one TMA copy as 9 blocks of 64 dims,
// each block P token rows x 128 bytes (128-byte swizzle).  Swap-AB keeps every MMA row
// a real token or value dim (the 16 heads are the N dimension):
//   S^T[64 tokens x 16 heads]  = K[64 x 576] . Q^T             (M 64, N 16, 36 K-steps)
//   O^T[512 dims x 16 heads] += V^T[512 x P] . P^T[P x 16]      (4 x M 128, N 16, P/16 K-steps)
// K is a K-major operand of the tile; V^T is the same tile read as an MN-major operand
// (64 consecutive dims per 128-byte row, token rows in groups of 8), so the value is
// never copied.  P^T is written by the softmax warps as a K-major operand (one 128-byte
// row of 64 tokens per head).  Q arrives by TMA too (16 head rows of the request).
//
// Warp roles (192 threads, one CTA per SM): warps 0-3 run the softmax and the epilogue,
// each on its 32-lane TMEM sub-partition (S^T with M = 64 keeps token 16w + l in lane
// 32w + l, l < 16; O^T keeps dim 128j + 32w + l in lane 32w + l); warp 4 resolves the
// chunk's tiles (selection -> page table) and issues the TMA copies into a ring of
// half-page tiles; one thread of warp 5 issues the MMAs.  Pipeline per tile i: TMA ->
// MMA1(i) into S buffer i % 2 -> softmax(i) writes P buffer i % 2 -> MMA2(i) accumulates O
// and frees the stage; MMA1(i+1) runs while softmax(i) does.  The softmax reads S^T from
// TMEM token-major, transposes it through shared memory and works head-major: thread t
// owns head t / 8 and 8 of the tile's tokens, so a head's max is 3 shuffles among 8 lanes
// and its P segment one 16-byte store.  The running max per head is raised only when a
// tile's max exceeds it by 2^8 (exp2 units); the warps then exchange the heads' factors
// and rescale O in TMEM.  Waiting threads sleep in mbarrier try_wait rather than spin.
//
// Work: the rows' selected pages form one flat list cut into W contiguous chunks, one
// per CTA; a CTA writes one partial (unnormalised O, max, sum) per row it touches at
// slot row + chunk, merged by k_merge with the log-sum-exp rule.  Value rows of tokens
// past the request's length are zeroed in shared memory before the P.V product, so NaN
// in unused slots cannot leak.  Every wait is bounded; a wait that runs out sets
// VX_DATA_TIMEOUT, drains the copies and MMAs in flight, frees the tensor memory and
// leaves the chunk's rows empty.
#include "vx_internal.h"
#include "vx_umma.cuh"

namespace vx {

constexpr int UM_THREADS = 192;
constexpr int UM_PROD_WARP = 4, UM_MMA_WARP = 5;
constexpr int UM_ROWS = 64;                                // MMA M of the score product
constexpr int UM_DQK = 576, UM_DV = 512, UM_KB = UM_DQK / 64;
constexpr int UM_QBYTES = 16 * UM_KB * 128;                // 18,432: 16 head rows x 576
constexpr int UM_QBLOCK = 16 * 128;                        // one 64-dim block of Q
constexpr int UM_PBYTES = 16 * 128;                        // 16 head rows x 64 tokens
constexpr uint32_t UM_TMEM_COLS = 128;
constexpr uint32_t UM_O_COL = 0;                           // O^T: 4 x 16 columns
constexpr uint32_t UM_S_COL = 64;                          // S^T: 2 buffers x 16 columns
constexpr float UM_RAISE_LOG2 = 8.f;
constexpr uint32_t UM_IDESC_S = umma_idesc_bf16(64, 16, false, false);
constexpr uint32_t UM_IDESC_O = umma_idesc_bf16(128, 16, true, false);
// Tokens per tile TR: 64 (a whole 64-token page) in a 2-stage ring, or 32 (a 32-token page,
// or half a 64-token one) in a 4-stage ring.  A tile's block b holds TR token rows at
// b * TR * 128 bytes; the score MMA reads M = 64 rows, so for TR = 32 rows 32..63 come from
// the next block (or, for the last block, the stage's slack) and are masked.  Measured on
// the MLA workload (decode + merge per call): 20.8 us with TR = 64 against 24.2 us with
// TR = 32; the per-tile MMA issue and hand-offs outweigh the finer ring.
template <int TR>
struct UmTile {
    static constexpr int STAGES = TR == 32 ? 4 : 2;  // as many as shared memory holds
    static constexpr uint32_t BS = TR * 128;                                         // one 64-dim block
    static constexpr uint32_t STAGE = ((UM_KB * BS + (UM_ROWS - TR) * 128) + 1023) & ~1023u;  // + read slack
    static constexpr uint32_t DATA = STAGES * STAGE + 2 * UM_QBYTES + 2 * UM_PBYTES;
};

struct UmMeta {
    int32_t row;     // -1: end of the chunk
    int32_t nvalid;  // valid tokens of the page
    int32_t qbuf;    // Q buffer holding this row's query
    int32_t pad;
};

template <int STAGES>
struct UmShared {
    unsigned long long kfull[STAGES], kfree[STAGES];
    unsigned long long sfull[2], sfree[2], pfull[2], pfree[2];
    unsigned long long xbar, drain;
    UmMeta meta[STAGES];
    float s_t[2][16][64];  // S of a tile, [head][token] (double buffered)
    float alpha[2][16];    // per-head rescale factors of a tile (double buffered)
    uint32_t tmem_base;
    volatile int32_t abort;
};

__device__ __forceinline__ Resolved resolve_page(const DecodeArgs &a, int64_t u, int64_t u_end) {
    Resolved rs{0, 0, 0, 0, false};
    if (u >= u_end) return rs;
    const int64_t r = u / a.units_per_row;  // one KV head: row == request
    const int64_t rem = u - r * a.units_per_row;
    const int i = static_cast<int>(rem / a.tiles_per_page);
    const int sub = static_cast<int>(rem - (int64_t)i * a.tiles_per_page);
    const int b = static_cast<int>(r);
    rs.row = static_cast<int32_t>(r);
    const int32_t L = a.seq_lens[b];
    if (L < 1 || L > a.max_pages * a.P) return rs;
    const int32_t j = a.sel[r * a.k + i];
    if (j < 0) return rs;
    const int n = ceil_div(L, a.P);
    if (j >= n) {
        set_err(a.err, VX_DATA_BAD_SELECTION);
        return rs;
    }
    const int32_t phys = a.page_indices[a.page_ptr[b] + j];
    if (phys < 0 || phys >= a.num_pool_pages) {
        set_err(a.err, VX_DATA_BAD_PAGE_ID);
        return rs;
    }
    const int tr = a.P / a.tiles_per_page;  // tokens per tile
    const int nvalid = min(tr, L - j * a.P - sub * tr);
    if (nvalid <= 0) return rs;
    rs.z = phys;
    rs.y = sub * tr;
    rs.nvalid = nvalid;
    rs.valid = true;
    return rs;
}

// Bounded wait on an mbarrier phase that also gives up once another thread of the CTA has
// given up (shared abort flag); a wait that runs out itself raises the flag.  The waiting
// threads sleep in try_wait (woken when the phase completes) instead of spinning: the warps
// of a role share the SM's schedulers with the softmax warps, whose issue slots a spinning
// waiter would take.
__device__ __forceinline__ bool um_wait(uint32_t bar, unsigned parity, volatile int32_t *abort) {
    if (mbar_test_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait_hint(bar, parity, 1000u)) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > WAIT_LIMIT_NS) {
            *abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int TR>
__global__ void __launch_bounds__(UM_THREADS, 1)
    k_decode_mla(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                 const DecodeArgs a) {
    using T = UmTile<TR>;
    constexpr int UM_STAGES = T::STAGES;
    constexpr uint32_t UM_STAGE_BYTES = T::STAGE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sStage = base;                                    // UM_STAGES tiles
    const uint32_t sQ = base + UM_STAGES * UM_STAGE_BYTES;           // 2 query buffers
    const uint32_t sP = sQ + 2 * UM_QBYTES;                          // 2 probability buffers
    UmShared<UM_STAGES> &sh = *reinterpret_cast<UmShared<UM_STAGES> *>(smem_raw + (base - raw) + T::DATA);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int64_t c = blockIdx.x;
    if (c >= a.chunks) return;
    const int64_t u_begin = chunk_start(c, a.units, a.chunks);
    const int64_t u_end = chunk_start(c + 1, a.units, a.chunks);
    const int64_t row_first = u_begin / a.units_per_row;
    const int64_t row_last = (u_end - 1) / a.units_per_row;
    constexpr uint32_t bs = T::BS;  // bytes of one 64-dim block of a tile

    if (tid == 0) {
        for (int s = 0; s < UM_STAGES; ++s) {
            mbar_init(smem_u32(&sh.kfull[s]), 1);
            mbar_init(smem_u32(&sh.kfree[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&sh.sfull[b]), 1);
            mbar_init(smem_u32(&sh.sfree[b]), 4);
            mbar_init(smem_u32(&sh.pfull[b]), 4);
            mbar_init(smem_u32(&sh.pfree[b]), 1);
        }
        mbar_init(smem_u32(&sh.xbar), 4);
        mbar_init(smem_u32(&sh.drain), 1);
        sh.abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&sh.tmem_base), UM_TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == UM_PROD_WARP && lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmQ);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int32_t *abort = &sh.abort;
    pdl_wait();  // the selection comes from the previous kernel on the stream

    if (warp == UM_PROD_WARP) {
        // ---------------------------------------------------------------- producer
        int64_t batch = u_begin;
        Resolved rs = resolve_page(a, batch + lane, u_end);
        uint32_t pending = __ballot_sync(FULL, rs.valid);
        uint32_t it = 0;
        int64_t qrow = -1;
        int32_t qsel = 1;
        bool ended = false;  // the end marker is posted
        for (;;) {
            while (pending == 0) {
                batch += 32;
                if (batch >= u_end) break;
                rs = resolve_page(a, batch + lane, u_end);
                pending = __ballot_sync(FULL, rs.valid);
            }
            const int st = static_cast<int>(it % UM_STAGES);
            if (it >= UM_STAGES &&
                !__all_sync(FULL, um_wait(smem_u32(&sh.kfree[st]), ((it / UM_STAGES) - 1) & 1u, abort)))
                break;
            if (pending == 0) {  // end marker
                if (lane == 0) {
                    sh.meta[st].row = -1;
                    sh.meta[st].nvalid = 0;
                    mbar_arrive(smem_u32(&sh.kfull[st]));
                }
                __syncwarp();
                ended = true;
                break;
            }
            const int src = __ffs(pending) - 1;
            pending &= pending - 1;
            const int32_t row = __shfl_sync(FULL, rs.row, src);
            const int32_t z = __shfl_sync(FULL, rs.z, src);
            const int32_t y = __shfl_sync(FULL, rs.y, src);
            const int32_t nv = __shfl_sync(FULL, rs.nvalid, src);
            const bool newq = row != qrow;
            if (newq) {
                qrow = row;
                qsel ^= 1;
            }
            if (lane == 0) {
                sh.meta[st].row = row;
                sh.meta[st].nvalid = nv;
                sh.meta[st].qbuf = qsel;
                const uint32_t bar = smem_u32(&sh.kfull[st]);
                mbar_arrive_expect_tx(bar, static_cast<uint32_t>(UM_KB) * bs + (newq ? UM_QBYTES : 0u));
                tma_load_4d(sStage + (uint32_t)st * UM_STAGE_BYTES, &tmK, 0, y, 0, z, bar);
                if (newq) tma_load_3d(sQ + (uint32_t)qsel * UM_QBYTES, &tmQ, 0, row * a.Hq, 0, bar);
            }
            __syncwarp();
            ++it;
        }
        // every issued copy lands before the CTA can exit (time-bounded, even after an abort).
        // Once the end marker is posted, tile it - UM_STAGES has landed (its stage's P.V product
        // was awaited) and that stage's barrier has moved on to the marker's phase, so only the
        // UM_STAGES - 1 tiles after it are awaited; after an abort the last UM_STAGES tiles are.
        const uint32_t inflight = ended ? (uint32_t)UM_STAGES - 1u : (uint32_t)UM_STAGES;
        for (uint32_t t = it > inflight ? it - inflight : 0; t < it; ++t)
            if (!mbar_wait_bounded(smem_u32(&sh.kfull[t % UM_STAGES]), (t / UM_STAGES) & 1u) && lane == 0)
                set_err(a.err, VX_DATA_TIMEOUT);
    } else if (warp == UM_MMA_WARP) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t n1 = 0, n2 = 0, end_at = 0xffffffffu;
            int32_t row_prev = -1;
            bool issued = false;
            unsigned long long t0 = globaltimer();
            uint32_t idle = 0;
            for (;;) {
                bool prog = false;
                if (n1 < end_at && n1 < n2 + 2) {
                    const int st = static_cast<int>(n1 % UM_STAGES);
                    if (mbar_test_wait(smem_u32(&sh.kfull[st]), (n1 / UM_STAGES) & 1u) &&
                        (n1 < 2 || mbar_test_wait(smem_u32(&sh.sfree[n1 & 1]), ((n1 >> 1) - 1) & 1u))) {
                        const volatile UmMeta *vm = &sh.meta[st];
                        const int32_t m_row = vm->row, m_qbuf = vm->qbuf;
                        if (m_row < 0) {
                            end_at = n1;
                            mbar_arrive(smem_u32(&sh.sfull[n1 & 1]));
                        } else {
                            tc_fence_after();
                            const uint32_t d = tmem + UM_S_COL + 16u * (n1 & 1);
                            // descriptors of the first K step; later steps advance the start
                            // address field (16-byte units, no carry: addresses < 256 KB)
                            const uint64_t da = umma_sdesc(sStage + (uint32_t)st * UM_STAGE_BYTES, 16u, 1024u);
                            const uint64_t db = umma_sdesc(sQ + (uint32_t)m_qbuf * UM_QBYTES, 16u, 1024u);
#pragma unroll
                            for (int blk = 0; blk < UM_KB; ++blk)
#pragma unroll
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_bf16_ss(d, da + ((blk * bs + kk * 32u) >> 4),
                                                 db + ((uint32_t)(blk * UM_QBLOCK + kk * 32) >> 4), UM_IDESC_S,
                                                 (blk | kk) ? 1u : 0u);
                            umma_commit(smem_u32(&sh.sfull[n1 & 1]));
                            issued = true;
                        }
                        ++n1;
                        prog = true;
                    }
                }
                if (n2 < n1 && n2 < end_at) {
                    if (mbar_test_wait(smem_u32(&sh.pfull[n2 & 1]), (n2 >> 1) & 1u)) {
                        tc_fence_after();
                        const int st = static_cast<int>(n2 % UM_STAGES);
                        const int32_t row = *const_cast<volatile int32_t *>(&sh.meta[st].row);
                        const bool first = row != row_prev;
                        row_prev = row;
                        const uint64_t da = umma_sdesc(sStage + (uint32_t)st * UM_STAGE_BYTES, bs, 1024u);
                        const uint64_t db = umma_sdesc(sP + (n2 & 1) * UM_PBYTES, 16u, 1024u);
                        constexpr int ksteps = TR / 16;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
#pragma unroll 4
                            for (int kk = 0; kk < ksteps; ++kk)
                                umma_bf16_ss(tmem + UM_O_COL + 16u * j, da + ((2u * j * bs + (uint32_t)kk * 2048u) >> 4),
                                             db + (uint32_t)kk * 2u, UM_IDESC_O, (first && kk == 0) ? 0u : 1u);
                        umma_commit(smem_u32(&sh.kfree[st]));
                        umma_commit(smem_u32(&sh.pfree[n2 & 1]));
                        ++n2;
                        prog = true;
                    }
                }
                if (n2 == end_at) break;
                if (prog) {
                    idle = 0;
                    continue;
                }
                // nothing to issue: back off briefly and poll both events again (a thread asleep
                // on one barrier would miss the other completing)
                __nanosleep(32);
                if (++idle == 1) t0 = globaltimer();
                if ((idle & 255u) == 0) {
                    if (*abort) break;
                    if (globaltimer() - t0 > WAIT_LIMIT_NS) {
                        *abort = 1;
                        break;
                    }
                }
            }
            if (issued) {  // every MMA this thread issued is done before the tensor memory is freed
                umma_commit(smem_u32(&sh.drain));
                if (!mbar_wait_bounded(smem_u32(&sh.drain), 0u)) set_err(a.err, VX_DATA_TIMEOUT);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax + epilogue (warps 0-3)
        // S^T is read from TMEM token-major (lane l < 16 of warp w: token 16w + l, 16 heads),
        // transposed through shared memory, and processed head-major: thread tid owns head
        // hh = tid / 8 and tokens 8 * (tid % 8) .. + 8 of the tile, so a head's running max and
        // sum live in the 8 lanes of one warp and its P row segment is one 16-byte store.
        const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
        const int tok = 16 * warp + lane;  // token of this lane in the S^T tile (lanes 0-15)
        const int hh = tid >> 3, part = tid & 7;
        int64_t cur_row = -1, flushed_to = row_first - 1;
        float m_run = -INFINITY, l_run = 0.f;  // head hh: running max (log2 units), this lane's sum
        uint32_t xph = 0;  // phases of xbar this warp has waited for
        bool failed = false, first = true;
        uint32_t i = 0;

        auto write_empty = [&](int64_t r) {
            if (warp == 0 && lane < a.G) {
                float *ml = a.ml_part + ((r + c) * a.G + lane) * 2;
                ml[0] = -INFINITY;
                ml[1] = 0.f;
            }
        };
        auto exchange = [&]() -> bool {  // the four warps meet (bounded)
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.xbar));
            const bool ok = __all_sync(FULL, um_wait(smem_u32(&sh.xbar), xph & 1u, abort));
            ++xph;
            return ok;
        };
        // partial of row `r`, whose last tile in this chunk is tile e
        auto epilogue = [&](int64_t r, uint32_t e) -> bool {
            if (!__all_sync(FULL, um_wait(smem_u32(&sh.pfree[e & 1]), (e >> 1) & 1u, abort))) return false;
            tc_fence_after();
            const int64_t slot = r + c;
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                uint32_t o[16];
                tmem_ld16(tmem + lane_base + UM_O_COL + 16u * j, o);
                tmem_wait_ld();
                const int dim = 128 * j + 32 * warp + lane;
#pragma unroll
                for (int h = 0; h < 16; ++h)
                    if (h < a.G) a.o_part[(slot * a.G + h) * UM_DV + dim] = __uint_as_float(o[h]);
            }
            tc_fence_before();
            float l = l_run;
            l += __shfl_xor_sync(FULL, l, 1);
            l += __shfl_xor_sync(FULL, l, 2);
            l += __shfl_xor_sync(FULL, l, 4);
            if (part == 0 && hh < a.G) {
                float *ml = a.ml_part + (slot * a.G + hh) * 2;
                ml[0] = m_run;
                ml[1] = l;
            }
            return true;
        };

        for (;; ++i) {
            if (!__all_sync(FULL, um_wait(smem_u32(&sh.sfull[i & 1]), (i >> 1) & 1u, abort))) {
                failed = true;
                break;
            }
            const int st = static_cast<int>(i % UM_STAGES);
            // the tile's metadata: acquire it from the producer's barrier (complete already;
            // its next phase needs this tile's P.V product, so it cannot have moved on)
            if (!__all_sync(FULL, um_wait(smem_u32(&sh.kfull[st]), (i / UM_STAGES) & 1u, abort))) {
                failed = true;
                break;
            }
            const int32_t row = *const_cast<volatile int32_t *>(&sh.meta[st].row);
            const int32_t nvalid = *const_cast<volatile int32_t *>(&sh.meta[st].nvalid);
            if (row < 0) break;
            if (row != cur_row) {
                if (cur_row >= 0) {
                    if (!epilogue(cur_row, i - 1)) {
                        failed = true;
                        break;
                    }
                    flushed_to = cur_row;
                }
                for (int64_t r = flushed_to + 1; r < row; ++r) write_empty(r);
                flushed_to = row - 1;
                cur_row = row;
                m_run = -INFINITY;
                l_run = 0.f;
                first = true;
            }
            // S^T of this warp's 16 tokens -> shared memory [head][token] (buffer i % 2)
            float *sS = &sh.s_t[i & 1][0][0];
            {
                tc_fence_after();
                uint32_t sr[16];
                tmem_ld16(tmem + lane_base + UM_S_COL + 16u * (i & 1), sr);
                tmem_wait_ld();
                tc_fence_before();
                if (lane < 16) {
#pragma unroll
                    for (int h = 0; h < 16; ++h) sS[h * 64 + tok] = __uint_as_float(sr[h]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sh.sfree[i & 1]));
            }
            if (!exchange()) {
                failed = true;
                break;
            }
            // head hh, tokens 8 * part .. + 8
            float x[8];
            {
                const float4 v0 = *reinterpret_cast<const float4 *>(sS + hh * 64 + part * 8);
                const float4 v1 = *reinterpret_cast<const float4 *>(sS + hh * 64 + part * 8 + 4);
                const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = part * 8 + e < nvalid ? vv[e] * a.scale_log2 : -INFINITY;
            }
            float mt = x[0];
#pragma unroll
            for (int e = 1; e < 8; ++e) mt = fmaxf(mt, x[e]);
            mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 1));
            mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 2));
            mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 4));
            // raise the running max only when the tile's exceeds it by 2^8 (exp2 units)
            const bool up = mt > m_run + UM_RAISE_LOG2;
            const float alpha = up ? exp2f(m_run - mt) : 1.f;
            if (up) m_run = mt;
            l_run *= alpha;
            if (!first) {
                // every dim of O needs the factor of every head: publish them, meet, and rescale
                // O in TMEM (once the previous tile's P.V product has landed) if any head rose
                if (part == 0) sh.alpha[i & 1][hh] = alpha;
                if (!exchange()) {
                    failed = true;
                    break;
                }
                const float4 *al = reinterpret_cast<const float4 *>(&sh.alpha[i & 1][0]);
                float af[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 v = al[q4];
                    af[4 * q4] = v.x;
                    af[4 * q4 + 1] = v.y;
                    af[4 * q4 + 2] = v.z;
                    af[4 * q4 + 3] = v.w;
                }
                bool any = false;
#pragma unroll
                for (int h = 0; h < 16; ++h) any |= af[h] != 1.f;
                if (any) {
                    if (!__all_sync(FULL, um_wait(smem_u32(&sh.pfree[(i - 1) & 1]), ((i - 1) >> 1) & 1u, abort))) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
#pragma unroll 1
                    for (int j = 0; j < 4; ++j) {
                        uint32_t o[16];
                        tmem_ld16(tmem + lane_base + UM_O_COL + 16u * j, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < 16; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * af[h]);
                        tmem_st16(tmem + lane_base + UM_O_COL + 16u * j, o);
                    }
                    tmem_wait_st();
                }
            }
            // P buffer i % 2 is free once the P.V product of tile i - 2 is done
            if (i >= 2 &&
                !__all_sync(FULL, um_wait(smem_u32(&sh.pfree[i & 1]), ((i >> 1) - 1) & 1u, abort))) {
                failed = true;
                break;
            }
            {
                // P row hh, tokens 8 * part .. + 8: one 16-byte chunk (128-byte swizzle)
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const float p0 = exp2f(x[e] - m_run), p1 = exp2f(x[e + 1] - m_run);
                    const __nv_bfloat162 pv = __floats2bfloat162_rn(p0, p1);
                    l_run += __low2float(pv) + __high2float(pv);
                    w4[e >> 1] = *reinterpret_cast<const uint32_t *>(&pv);
                }
                const uint32_t addr = sP + (i & 1) * UM_PBYTES + hh * 128 + ((uint32_t)(part ^ (hh & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w4[0]), "r"(w4[1]),
                             "r"(w4[2]), "r"(w4[3])
                             : "memory");
            }
            if (nvalid < TR) {
                // value rows of the tokens past the length: zero (blocks 0-7, 128 bytes each)
                const uint32_t sK = sStage + (uint32_t)st * UM_STAGE_BYTES;
                const int n16 = (TR - nvalid) * 64;  // 16-byte pieces
                for (int idx = tid; idx < n16; idx += 128) {
                    const int t = nvalid + (idx >> 6), blk = (idx >> 3) & 7, piece = idx & 7;
                    const uint32_t addr = sK + (uint32_t)blk * bs + (uint32_t)t * 128u + (uint32_t)piece * 16u;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
                }
            }
            fence_proxy_async_smem();  // P and the zeroed rows are read by the tensor cores
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.pfull[i & 1]));
            first = false;
        }
        if (!failed && cur_row >= 0) {
            if (epilogue(cur_row, i - 1))
                flushed_to = cur_row;
            else
                failed = true;
        }
        if (failed) {
            if (tid == 0) set_err(a.err, VX_DATA_TIMEOUT);
            for (int64_t r = row_first; r <= row_last; ++r) write_empty(r);
        } else {
            for (int64_t r = flushed_to + 1; r <= row_last; ++r) write_empty(r);
        }
    }

    // teardown: every role has drained its copies, MMAs and TMEM reads
    if (tid == 0 && sh.abort) set_err(a.err, VX_DATA_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, UM_TMEM_COLS);
    }
}

template <int TR>
static cudaError_t launch_decode_mla_tr(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmQ, int grid,
                                       cudaStream_t s, bool pdl) {
    using T = UmTile<TR>;
    const size_t smem = 1024 + (size_t)T::DATA + sizeof(UmShared<T::STAGES>);
    static std::atomic<unsigned long long> done;
    cudaError_t e = ensure_smem_limit(k_decode_mla<TR>, (int)smem, done);
    if (e != cudaSuccess) return e;
    return launch_k(k_decode_mla<TR>, dim3(grid), dim3(UM_THREADS), smem, s, pdl, tmK, tmQ, a);
}

// tile height = page_size / tiles_per_page (the TMA box the host encoded): 64 or 32 tokens
cudaError_t launch_decode_mla(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmQ, int grid,
                              cudaStream_t s, bool pdl) {
    const int tr = a.P / a.tiles_per_page;
    if (tr == 64) return launch_decode_mla_tr<64>(a, tmK, tmQ, grid, s, pdl);
    if (tr == 32) return launch_decode_mla_tr<32>(a, tmK, tmQ, grid, s, pdl);
    return cudaErrorInvalidValue;
}

}  // namespace vx
