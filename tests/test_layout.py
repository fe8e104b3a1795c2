"""Host-side checks of the packed weight layout the tensor-core kernels read.

The library stores each weight matrix as 128-row x 64-column bf16 tiles in the
exact shared-memory image of the 128-byte swizzle (16-byte chunk c of row r at
chunk c ^ (r % 8)), tiles grouped in pairs that one 32 KB bulk copy moves:
(gate, up) of a 128-row block, or two adjacent 128-row blocks of W_down with a
zero-filled odd half.  The offset helpers in csrc/layer.h define that layout for
the pack kernel and the kernels' address arithmetic; this test compiles them
with the host compiler and checks that they are bijections onto the packed
buffers with the pair structure described above.
"""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

PROGRAM = r"""
#include "layer.h"
#include <cstdio>
#include <vector>

static int fails = 0;
#define CHECK(c, ...) do { if (!(c)) { ++fails; if (fails < 10) std::printf(__VA_ARGS__); } } while (0)

int main() {
    using namespace moe;
    // 1. the swizzle inside one tile is a bijection on its 8192 elements, and chunk c
    //    of row r lands in chunk c ^ (r % 8) of that row
    {
        std::vector<int> hit(8192, 0);
        for (int r = 0; r < 128; ++r)
            for (int c = 0; c < 64; ++c) {
                const size_t o = swizzled_in_tile(r, c);
                CHECK(o < 8192, "tile offset out of range %d %d\n", r, c);
                if (o < 8192) ++hit[o];
                CHECK(o / 64 == (size_t)r, "row moved %d %d\n", r, c);
                CHECK((o % 64) / 8 == (size_t)((c / 8) ^ (r % 8)), "chunk %d %d\n", r, c);
                CHECK(o % 8 == (size_t)(c % 8), "element in chunk %d %d\n", r, c);
            }
        for (int i = 0; i < 8192; ++i) CHECK(hit[i] == 1, "tile slot %d hit %d times\n", i, hit[i]);
    }
    // 2. gate/up pairs: a bijection of (expert, row, column, which) onto E*I*H*2
    //    elements; gate and up of the same (row, column) sit one tile (8192) apart
    {
        const int E = 3, I = 256, H = 192;
        std::vector<int> hit((size_t)E * I * H * 2, 0);
        for (int e = 0; e < E; ++e)
            for (int r = 0; r < I; ++r)
                for (int c = 0; c < H; ++c) {
                    const size_t g = packed_gu_offset(e, r, c, 0, I, H);
                    const size_t u = packed_gu_offset(e, r, c, 1, I, H);
                    CHECK(u == g + 8192, "gate/up not adjacent %d %d %d\n", e, r, c);
                    CHECK(u < hit.size(), "gate/up offset out of range\n");
                    if (u < hit.size()) { ++hit[g]; ++hit[u]; }
                    // a tile pair is 32 KB-contiguous and pairs run expert, row block, k-block
                    const size_t pair = g / 16384;
                    const size_t want = ((size_t)e * (I / 128) + r / 128) * (H / 64) + c / 64;
                    CHECK(pair == want, "pair order %d %d %d\n", e, r, c);
                }
        for (size_t i = 0; i < hit.size(); ++i) CHECK(hit[i] == 1, "gu slot %zu hit %d\n", i, hit[i]);
    }
    // 3. down pairs with an odd number of 128-row blocks: injective into the padded
    //    buffer, and the slots left over are exactly the zero-filled odd half
    {
        const int E = 2, H = 384, I = 128;                // 3 row blocks -> 2 pairs
        const size_t n = packed_down_elems(E, H, I);
        CHECK(n == (size_t)E * 2 * (I / 64) * 2 * 8192, "padded size %zu\n", n);
        std::vector<int> hit(n, 0);
        for (int e = 0; e < E; ++e)
            for (int r = 0; r < H; ++r)
                for (int c = 0; c < I; ++c) {
                    const size_t o = packed_down_offset(e, r, c, H, I);
                    CHECK(o < n, "down offset out of range\n");
                    if (o < n) ++hit[o];
                    if (r < 256) {
                        // rows r and r + 128 of the same pair are one tile apart
                        const int r2 = r ^ 128;
                        if (r2 < H)
                            CHECK((o / 8192) / 2 == packed_down_offset(e, r2, c, H, I) / 8192 / 2,
                                  "down pair split %d %d %d\n", e, r, c);
                    }
                }
        size_t empty = 0;
        for (size_t i = 0; i < n; ++i) {
            CHECK(hit[i] <= 1, "down slot %zu hit %d\n", i, hit[i]);
            empty += hit[i] == 0;
        }
        CHECK(empty == n - (size_t)E * H * I, "zero fill %zu\n", empty);
        // the empty slots are whole tiles: the second tile of each expert's last pair
        for (int e = 0; e < E; ++e)
            for (int kb = 0; kb < I / 64; ++kb) {
                const size_t tile = ((((size_t)e * 2 + 1) * (I / 64) + kb) * 2 + 1);
                for (int i = 0; i < 8192; ++i) CHECK(hit[tile * 8192 + i] == 0, "fill tile\n");
            }
    }
    std::printf(fails ? "FAIL %d\n" : "OK\n", fails);
    return fails ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.isdir(CUDA_INC),
                    reason="needs g++ and the CUDA headers")
def test_packed_layout_helpers():
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "layout.cpp")
        exe = os.path.join(d, "layout")
        with open(src, "w") as f:
            f.write(PROGRAM)
        subprocess.run(["g++", "-std=c++17", "-O1", "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "sparse_moe_transformer_b200", "csrc"),
                        "-I", CUDA_INC, src, "-o", exe], check=True)
        r = subprocess.run([exe], capture_output=True, text=True)
        assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout
