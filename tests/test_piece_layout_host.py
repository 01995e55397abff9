"""The decode split's piece layout (piece_start / piece_of in csrc/vx_internal.h), checked on the
host: compiled with nvcc into a small host program that builds layouts the way the planner does
(one even chunk per warp, plus late pieces over the last DEC_DYN_PCT% of the tiles when a warp's
share allows them) and checks, for many shapes, the properties the decode and merge kernels rely
on: pieces are non-empty, contiguous and in unit order; piece_of inverts piece_start; slot
(row + piece) is unique over every (row, piece) pair that shares a tile; a row's pieces are the
contiguous run piece_of(first tile) .. piece_of(last tile); and that run never exceeds the
merge launcher's bound on partials per row."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_block_sparse_kv_b200", "csrc")

PROGRAM = r"""
#include "vx_internal.h"
#include <cstdio>
#include <vector>
#include <algorithm>

using namespace vx;

// the planner's layout for a planned GQA split (mirrors plan() in vx_api.cu)
static void layout(int64_t T, int sms, int64_t &Us, int64_t &Ws, int64_t &W) {
    int64_t w = std::min<int64_t>((int64_t)sms * DEC_WARPS, T);
    int64_t us = T, wd = 0;
    const int64_t piece = T / w / DEC_DYN_DIV;
    const int64_t ud = T * DEC_DYN_PCT / 100;
    wd = piece >= DEC_DYN_MIN_PIECE ? ud / piece : 0;
    if (wd >= 1 && T - ud >= w) us = T - ud; else wd = 0;
    Us = us; Ws = w; W = w + wd;
}

int main() {
    long checked = 0, with_late = 0;
    const int sms_list[] = {1, 2, 7, 132, 148};
    const int64_t rows_list[] = {1, 3, 16, 64, 256, 1280, 2048};
    const int64_t upr_list[] = {1, 5, 8, 32, 64, 128, 160, 256};
    for (int sms : sms_list)
        for (int64_t rows : rows_list)
            for (int64_t upr : upr_list) {
                const int64_t T = rows * upr;
                int64_t Us, Ws, W;
                layout(T, sms, Us, Ws, W);
                if (W > Ws) ++with_late;
                std::vector<int64_t> st(W + 1);
                for (int64_t c = 0; c <= W; ++c) st[c] = piece_start(c, T, Us, Ws, W);
                if (st[0] != 0 || st[W] != T) { printf("FAIL ends T=%lld\n", (long long)T); return 1; }
                for (int64_t c = 0; c < W; ++c)
                    if (st[c + 1] <= st[c]) { printf("FAIL empty piece %lld T=%lld W=%lld\n", (long long)c, (long long)T, (long long)W); return 1; }
                for (int64_t c = 0; c < W; ++c)
                    for (int64_t u : {st[c], st[c + 1] - 1, (st[c] + st[c + 1]) / 2})
                        if (piece_of(u, T, Us, Ws, W) != c) { printf("FAIL piece_of u=%lld\n", (long long)u); return 1; }
                std::vector<char> used(rows + W, 0);
                for (int64_t c = 0; c < W; ++c)
                    for (int64_t r = st[c] / upr; r <= (st[c + 1] - 1) / upr; ++r) {
                        const int64_t slot = r + c;
                        if (slot >= rows + W || used[slot]) { printf("FAIL slot %lld\n", (long long)slot); return 1; }
                        used[slot] = 1;
                    }
                // the merge launcher's bound on partials per row
                int64_t np_max = (upr * Ws + Us - 1) / Us + 1;
                if (W > Ws) np_max += (upr * (W - Ws) + (T - Us) - 1) / (T - Us) + 1;
                for (int64_t r = 0; r < rows; ++r) {
                    const int64_t lo = piece_of(r * upr, T, Us, Ws, W), hi = piece_of((r + 1) * upr - 1, T, Us, Ws, W);
                    for (int64_t c = lo; c <= hi; ++c)
                        if (!(st[c] < (r + 1) * upr && st[c + 1] > r * upr)) { printf("FAIL run r=%lld\n", (long long)r); return 1; }
                    if (lo > 0 && st[lo] > r * upr) { printf("FAIL run start r=%lld\n", (long long)r); return 1; }
                    if (hi - lo + 1 > np_max) { printf("FAIL np %lld > %lld\n", (long long)(hi - lo + 1), (long long)np_max); return 1; }
                }
                ++checked;
            }
    printf("ok %ld layouts, %ld with late pieces\n", checked, with_late);
    return with_late > 0 ? 0 : 2;
}
"""


def test_piece_layout_properties():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "piece_layout_check.cu")
        exe = os.path.join(d, "piece_layout_check")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                        "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True, capture_output=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stdout + r.stderr
        assert r.stdout.startswith("ok"), r.stdout
