// k_decode_mla.cu -- exact attention over the selected pages for the MLA geometry.
//
// Vortex paper note, section 系统设计 3: besides reusing dense attention backends the
// system adds its own kernel for more general MLA geometry; the MLA experiment section
// runs GLM-4.7-Flash (one shared latent KV per token: 512 latent + 64 rope dims; the
// first 512 dims are also the value).
//
// Geometry: 1 KV head, up to 16 query heads, Dqk = 576, Dv = 512.  The 16 heads fill the
// M dimension of mma.m16n8k16, so the contraction is a real dense tile:
//   S[16 heads x 32 tokens] = Q[16 x 576] . K^T       (36 k-steps x 4 n-tiles)
//   O[16 heads x 512 dims] += P[16 x 32] . V[32 x 512] (2 k-steps x 64 n-tiles)
// Work: the selected pages are cut into 32-token tiles; the rows' tiles form one flat
// list cut into W contiguous chunks, one chunk per 4-warp block (as in the GQA kernel,
// partials go to slot row + chunk and are merged with the log-sum-exp rule).  All four
// warps work on every tile: warp w contracts dims [144w, 144w+144) of Q.K^T for all 32
// tokens (four independent accumulation chains, one per 8-token n-tile), the four
// partial S tiles are summed through shared memory in a fixed order (so every warp holds
// the same S), each warp runs the same online softmax (skipping the output rescale when
// no row maximum moved) and then owns output dims [128w, 128w+128) of P.V.  K tiles
// (32 x 576 bf16, one TMA copy of 32 whole rows: 288 segments of 128 bytes, segment =
// token * 9 + 64-column block, 128-byte swizzle by segment index, so the 8 rows of an
// ldmatrix hit 8 distinct bank groups) stream through a MLA_STAGES-deep ring filled by
// one elected thread; a stage is refilled once every warp has passed the next tile's
// barrier.
#include "vx_internal.h"

namespace vx {

constexpr int MLA_THREADS = 128;
constexpr int MLA_STAGES = 2;
constexpr int MLA_DQK = 576, MLA_DV = 512;
constexpr int MLA_KB = MLA_DQK / 64;                   // 9 boxes per tile
constexpr int MLA_TILE = MLA_TILE_TOKENS * MLA_DQK * 2;  // 36 KB
constexpr int MLA_QBOX = 16 * 128;                     // Q: 16 head rows x 128 bytes
constexpr int MLA_QBYTES = MLA_KB * MLA_QBOX;          // 18 KB
constexpr int MLA_KSTEPS_PER_WARP = MLA_DQK / 16 / 4;  // 9
constexpr int MLA_SNT = MLA_TILE_TOKENS / 8;           // 4 n-tiles of tokens in S
constexpr int MLA_NT_PER_WARP = MLA_DV / 8 / 4;        // 16 n-tiles of output dims per warp

struct MlaMeta {
    int32_t row;  // -1: end of the chunk
    int32_t nvalid;
};

struct MlaShared {
    float4 s_part[2][4][MLA_SNT][32];  // partial S per warp and n-tile, per lane (double buffered)
    MlaMeta meta[MLA_STAGES];
    unsigned long long full[MLA_STAGES];
};

__device__ __forceinline__ Resolved resolve_mla(const DecodeArgs &a, int64_t u, int64_t u_end) {
    Resolved rs{0, 0, 0, 0, false};
    if (u >= u_end) return rs;
    const int64_t r = u / a.units_per_row;
    const int64_t rem = u - r * a.units_per_row;
    const int i = static_cast<int>(rem / a.tiles_per_page);
    const int sub = static_cast<int>(rem - (int64_t)i * a.tiles_per_page);
    const int b = static_cast<int>(r);  // one KV head: row == request
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
    const int tok0 = j * a.P + sub * MLA_TILE_TOKENS;
    const int nvalid = min(MLA_TILE_TOKENS, L - tok0);
    if (nvalid <= 0) return rs;
    const int32_t phys = a.page_indices[a.page_ptr[b] + j];
    if (phys < 0 || phys >= a.num_pool_pages) {
        set_err(a.err, VX_DATA_BAD_PAGE_ID);
        return rs;
    }
    rs.z = phys;
    rs.y = sub * MLA_TILE_TOKENS;
    rs.nvalid = nvalid;
    rs.valid = true;
    return rs;
}

// keep-mask of a packed bf16 pair holding tokens t and t + 1
__device__ __forceinline__ uint32_t pair_mask(int t, int nvalid) {
    return (t < nvalid ? 0x0000ffffu : 0u) | (t + 1 < nvalid ? 0xffff0000u : 0u);
}

__global__ void __launch_bounds__(MLA_THREADS, 2)
    k_decode_mla(const __grid_constant__ CUtensorMap tmK, const DecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sK0 = base;                           // MLA_STAGES tiles
    const uint32_t sQ = base + MLA_STAGES * MLA_TILE;    // 16 heads x 576, swizzled
    MlaShared &sh = *reinterpret_cast<MlaShared *>(smem_raw + (base - raw) + MLA_STAGES * MLA_TILE + MLA_QBYTES);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g4 = lane >> 2, q4 = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;

    const int64_t c = blockIdx.x;
    if (c >= a.chunks) return;
    const int64_t u_begin = chunk_start(c, a.units, a.chunks);
    const int64_t u_end = chunk_start(c + 1, a.units, a.chunks);
    const int64_t row_first = u_begin / a.units_per_row;
    const int64_t row_last = (u_end - 1) / a.units_per_row;
    if (tid == 0) {
        for (int s = 0; s < MLA_STAGES; ++s) mbar_init(smem_u32(&sh.full[s]), 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
    }
    __syncthreads();

    int64_t q_row = -1;  // row whose Q is staged in shared memory
    auto stage_q = [&](int64_t r) {
        // stage Q[16 heads][576] into shared memory in the swizzled box layout
        __syncthreads();  // nobody still reads the previous row's Q
        const __nv_bfloat16 *qb = a.q + (size_t)r * a.Hq * MLA_DQK;
        constexpr int QCH = 16 * (MLA_DQK / 8) / MLA_THREADS;  // 16-byte chunks per thread
        static_assert(16 * (MLA_DQK / 8) % MLA_THREADS == 0, "Q chunks split evenly");
        uint4 v[QCH];  // every load is issued before the first store
#pragma unroll
        for (int k = 0; k < QCH; ++k) {
            const int i = tid + k * MLA_THREADS;
            const int head = i / (MLA_DQK / 8), ch = i % (MLA_DQK / 8);
            v[k] = head < a.G ? __ldg(reinterpret_cast<const uint4 *>(qb + (size_t)head * MLA_DQK + ch * 8))
                              : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < QCH; ++k) {
            const int i = tid + k * MLA_THREADS;
            const int head = i / (MLA_DQK / 8), ch = i % (MLA_DQK / 8);
            const uint32_t dst = sQ + (ch >> 3) * MLA_QBOX + swz128(head, ch & 7);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(v[k].x), "r"(v[k].y),
                         "r"(v[k].z), "r"(v[k].w)
                         : "memory");
        }
        __syncthreads();
        q_row = r;
    };
    // Q of the chunk's first row is staged before waiting on the previous kernel: the query
    // is an input of the call, complete before this grid starts (the grid runs either in
    // plain stream order or after the top-k kernel, which itself starts after the scorer
    // ends).  Only the selection is written by the previous kernel.
    stage_q(row_first);
    pdl_wait();

    // ---- producer state (warp 0)
    int64_t batch = u_begin;
    Resolved rs{};
    uint32_t pending = 0;
    bool prod_done = false;
    if (warp == 0) {
        rs = resolve_mla(a, batch + lane, u_end);
        pending = __ballot_sync(FULL, rs.valid);
    }
    // issue the next valid tile into `st`, or the end marker; warp 0 only
    auto issue = [&](int st) {
        if (prod_done) return;
        while (pending == 0) {
            batch += 32;
            if (batch >= u_end) break;
            rs = resolve_mla(a, batch + lane, u_end);
            pending = __ballot_sync(FULL, rs.valid);
        }
        const uint32_t bar = smem_u32(&sh.full[st]);
        if (pending == 0) {
            if (lane == 0) {
                sh.meta[st].row = -1;
                sh.meta[st].nvalid = 0;
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
            }
            prod_done = true;
            __syncwarp();
            return;
        }
        const int src = __ffs(pending) - 1;
        pending &= pending - 1;
        const int32_t row = __shfl_sync(FULL, rs.row, src);
        const int32_t z = __shfl_sync(FULL, rs.z, src);
        const int32_t y = __shfl_sync(FULL, rs.y, src);
        const int32_t nv = __shfl_sync(FULL, rs.nvalid, src);
        if (lane == 0) {
            sh.meta[st].row = row;
            sh.meta[st].nvalid = nv;
            // no proxy fence: this stage's earlier shared-memory reads have completed,
            // their values were consumed before the barrier that released the stage
            mbar_arrive_expect_tx(bar, MLA_TILE);
            const uint32_t dst = sK0 + (uint32_t)st * MLA_TILE;
            tma_load_4d(dst, &tmK, 0, 0, y, z, bar);
        }
        __syncwarp();
    };
    if (warp == 0)
        for (int s = 0; s < MLA_STAGES; ++s) issue(s);

    // ---- consumer state (every warp)
    float acc[MLA_NT_PER_WARP][4];
    float m_run[2], l_run[2];
    int64_t cur_row = -1, flushed_to = row_first - 1;

    auto write_empty = [&](int64_t r) {
        if (warp == 0 && lane < a.G) {
            float *ml = a.ml_part + ((r + c) * a.G + lane) * 2;
            ml[0] = -INFINITY;
            ml[1] = 0.f;
        }
    };
    auto flush = [&](int64_t r) {
        const int64_t slot = r + c;
#pragma unroll
        for (int nt = 0; nt < MLA_NT_PER_WARP; ++nt)
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const int head = g4 + 8 * (e >> 1);
                const int dim = warp * 128 + nt * 8 + 2 * q4;
                if (head < a.G)
                    *reinterpret_cast<float2 *>(a.o_part + (slot * a.G + head) * MLA_DV + dim) =
                        make_float2(acc[nt][e], acc[nt][e + 1]);
            }
        float lt[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float v = l_run[i];
            v += __shfl_xor_sync(FULL, v, 1);
            v += __shfl_xor_sync(FULL, v, 2);
            lt[i] = v;
        }
        if (warp == 0 && q4 == 0) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int head = g4 + 8 * i;
                if (head < a.G) {
                    float *ml = a.ml_part + (slot * a.G + head) * 2;
                    ml[0] = m_run[i];
                    ml[1] = lt[i];
                }
            }
        }
    };
    auto start_row = [&](int64_t r) {
        if (r != q_row) stage_q(r);
#pragma unroll
        for (int nt = 0; nt < MLA_NT_PER_WARP; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.f;
    };

    // the first tile's Q if it is not row_first's (start_row would stage it otherwise)
    __syncthreads();  // the producer's first stage meta is visible
    if (sh.meta[0].row >= 0 && sh.meta[0].row != q_row) stage_q(sh.meta[0].row);

    bool failed = false;
    for (uint32_t it = 0;; ++it) {
        const int st = static_cast<int>(it % MLA_STAGES);
        const bool ok = __syncthreads_and(mbar_wait_bounded(smem_u32(&sh.full[st]), (it / MLA_STAGES) & 1u));
        if (!ok) {
            failed = true;
            break;
        }
        const int64_t row = sh.meta[st].row;
        const int nvalid = sh.meta[st].nvalid;
        if (row < 0) break;  // end of the chunk (uniform)
        if (row != cur_row) {
            if (cur_row >= 0) {
                flush(cur_row);
                flushed_to = cur_row;
            }
            for (int64_t r = flushed_to + 1; r < row; ++r) write_empty(r);
            flushed_to = row - 1;
            start_row(row);
            cur_row = row;
        }
        const uint32_t sK = sK0 + (uint32_t)st * MLA_TILE;
        const int buf = it & 1;

        // partial S over this warp's 144 dims, four 8-token n-tiles
        float s[MLA_SNT][4];
#pragma unroll
        for (int nt = 0; nt < MLA_SNT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < MLA_KSTEPS_PER_WARP; ++kk) {
            const int kg = warp * MLA_KSTEPS_PER_WARP + kk;  // global 16-dim step
            const int box = kg >> 2, c0 = (kg & 3) * 2;
            uint32_t qa0, qa1, qa2, qa3;
            ldsm_x4(sQ + box * MLA_QBOX + swz128(rr + 8 * (mi & 1), c0 + (mi >> 1)), qa0, qa1, qa2, qa3);
#pragma unroll
            for (int np = 0; np < MLA_SNT / 2; ++np) {  // pairs of token n-tiles
                uint32_t kb0, kb1, kb2, kb3;
                ldsm_x4(sK + swz128((np * 16 + rr + 8 * (mi >> 1)) * MLA_KB + box, c0 + (mi & 1)), kb0, kb1, kb2, kb3);
                mma_bf16_16816(s[2 * np], qa0, qa1, qa2, qa3, kb0, kb1);
                mma_bf16_16816(s[2 * np + 1], qa0, qa1, qa2, qa3, kb2, kb3);
            }
        }
#pragma unroll
        for (int nt = 0; nt < MLA_SNT; ++nt)
            sh.s_part[buf][warp][nt][lane] = make_float4(s[nt][0], s[nt][1], s[nt][2], s[nt][3]);
        __syncthreads();
        // the stage used by the previous tile is free now: refill it
        if (warp == 0 && it > 0) issue(static_cast<int>((it - 1) % MLA_STAGES));
        float x[MLA_SNT][4];
#pragma unroll
        for (int nt = 0; nt < MLA_SNT; ++nt) {
            float4 t = sh.s_part[buf][0][nt][lane];
#pragma unroll
            for (int w = 1; w < 4; ++w) {
                const float4 p = sh.s_part[buf][w][nt][lane];
                t.x += p.x;
                t.y += p.y;
                t.z += p.z;
                t.w += p.w;
            }
            x[nt][0] = t.x;
            x[nt][1] = t.y;
            x[nt][2] = t.z;
            x[nt][3] = t.w;
        }
        // online softmax over the 32 tokens (columns); rows = heads g4 and g4 + 8
#pragma unroll
        for (int nt = 0; nt < MLA_SNT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = nt * 8 + 2 * q4 + (e & 1);
                x[nt][e] = tok < nvalid ? x[nt][e] * a.scale_log2 : -INFINITY;
            }
        float alpha[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < MLA_SNT; ++nt) mx = fmaxf(mx, fmaxf(x[nt][2 * i], x[nt][2 * i + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
            const float m_new = fmaxf(m_run[i], mx);
            alpha[i] = exp2f(m_run[i] - m_new);
            m_run[i] = m_new;
        }
        float p[MLA_SNT][4];
#pragma unroll
        for (int nt = 0; nt < MLA_SNT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) p[nt][e] = exp2f(x[nt][e] - m_run[e >> 1]);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float add = 0.f;
#pragma unroll
            for (int nt = 0; nt < MLA_SNT; ++nt) add += p[nt][2 * i] + p[nt][2 * i + 1];
            l_run[i] = l_run[i] * alpha[i] + add;
        }
        if (__any_sync(FULL, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
            for (int nt = 0; nt < MLA_NT_PER_WARP; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][e] *= alpha[e >> 1];
        }
        // O[:, warp dims] += P . V over two 16-token k-steps; V = first 512 dims of the K rows
        const bool tail = nvalid < MLA_TILE_TOKENS;
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const uint32_t pa0 = pack_bf16x2(p[2 * ks][0], p[2 * ks][1]);
            const uint32_t pa1 = pack_bf16x2(p[2 * ks][2], p[2 * ks][3]);
            const uint32_t pa2 = pack_bf16x2(p[2 * ks + 1][0], p[2 * ks + 1][1]);
            const uint32_t pa3 = pack_bf16x2(p[2 * ks + 1][2], p[2 * ks + 1][3]);
            const uint32_t mlo = pair_mask(ks * 16 + 2 * q4, nvalid);
            const uint32_t mhi = pair_mask(ks * 16 + 8 + 2 * q4, nvalid);
#pragma unroll
            for (int pr = 0; pr < MLA_NT_PER_WARP / 2; ++pr) {
                const int ch = warp * 16 + pr * 2;  // 16-byte dim chunk of the first n-tile
                const int box = ch >> 3, cc = ch & 7;
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(sK + swz128((ks * 16 + rr + 8 * (mi & 1)) * MLA_KB + box, cc + (mi >> 1)), v0, v1, v2, v3);
                if (tail) {
                    v0 &= mlo;
                    v1 &= mhi;
                    v2 &= mlo;
                    v3 &= mhi;
                }
                mma_bf16_16816(acc[2 * pr], pa0, pa1, pa2, pa3, v0, v1);
                mma_bf16_16816(acc[2 * pr + 1], pa0, pa1, pa2, pa3, v2, v3);
            }
        }
    }

    if (failed) {
        if (tid == 0) set_err(a.err, VX_DATA_TIMEOUT);
        // let every issued load land before the block exits
        for (int s = 0; s < MLA_STAGES; ++s) (void)mbar_wait_bounded(smem_u32(&sh.full[s]), 0u);
        for (int64_t r = row_first; r <= row_last; ++r) write_empty(r);
        return;
    }
    if (cur_row >= 0) {
        flush(cur_row);
        flushed_to = cur_row;
    }
    for (int64_t r = flushed_to + 1; r <= row_last; ++r) write_empty(r);
}

cudaError_t launch_decode_mla(const DecodeArgs &a, const CUtensorMap &tmK, int grid, cudaStream_t s, bool pdl) {
    const size_t smem = 1024 + (size_t)MLA_STAGES * MLA_TILE + MLA_QBYTES + sizeof(MlaShared);
    static std::atomic<unsigned long long> done;
    cudaError_t e = ensure_smem_limit(k_decode_mla, (int)smem, done);
    if (e != cudaSuccess) return e;
    return launch_k(k_decode_mla, dim3(grid), dim3(MLA_THREADS), smem, s, pdl, tmK, a);
}

}  // namespace vx
