// Host-only dump of the tile list that the verify kernels walk for one (sequence, kv head), with
// the plan set up as the library's launch code sets it up (ripe_verify.cu: launch_single_loop,
// launch_draft and launch_verify_wave).  tests/test_tile_plan.py compiles it with nvcc and checks the tiles against
// the oracle's plane rule; nothing here runs on a GPU.
//
// Input, one case per line:
//   V T W B R max_T max_B mode nloops loop_0 .. loop_{nloops-1}
//     verification (nloops = 1: one call at loop_0; nloops > 1: a wavefront call whose block
//     position j sits at loop_{j mod nloops})
//   D T W R max_T max_B mode r j sink window
//     a draft step at block position j and loop r (launch_draft: the plan's block is positions
//     0..j, the query is position j; window = -1 for a full-context draft)
// Output per case: one line "kind t0 cnt y plane" per tile, then "E total".
#include <cstdio>

#include "ripe_common.cuh"

int main() {
    char what[4];
    while (std::scanf("%3s", what) == 1) {
        int T, W, B, R, max_T, max_B, mode, nloops = 1, sink = 0, dwin = -1, dj = 0;
        int loops[ripe::kMaxQueryRows];
        if (what[0] == 'V') {
            if (std::scanf("%d %d %d %d %d %d %d %d", &T, &W, &B, &R, &max_T, &max_B, &mode, &nloops) != 8) return 2;
            for (int k = 0; k < nloops; ++k)
                if (std::scanf("%d", &loops[k]) != 1) return 2;
        } else {
            if (std::scanf("%d %d %d %d %d %d %d %d %d %d", &T, &W, &R, &max_T, &max_B, &mode, &loops[0], &dj, &sink,
                           &dwin) != 10)
                return 2;
            B = dj + 1;
        }
        // cache geometry (ripe_cache_alloc)
        const int Wc = W > max_T ? max_T : W;
        const int ring_slots = Wc + max_B < max_T ? Wc + max_B : max_T;
        const int deep_rows = max_T - Wc;
        ripe::PlanArgs pa{};
        pa.W = Wc;
        pa.B = B;
        pa.R = R;
        pa.ring_slots = ring_slots;
        pa.deep_box = (deep_rows == 0 || deep_rows >= ripe::kTileRows) ? ripe::kTileRows : deep_rows;
        pa.ring_box = ring_slots < ripe::kTileRows ? ring_slots : ripe::kTileRows;
        pa.sink = sink;
        pa.dwin = dwin;
        pa.dj = dj;
        if (nloops == 1) {  // single loop: at the deepest loop the window rule changes nothing
            pa.mode_eff = (mode == RIPE_WINDOW_CACHE_RELATIVE || loops[0] == R - 1) ? 1 : 0;
            pa.nloops = 1;
            pa.loop[0] = static_cast<uint8_t>(loops[0]);
        } else {            // wavefront: the distinct loops of the block, in increasing order
            pa.mode_eff = mode == RIPE_WINDOW_CACHE_RELATIVE ? 1 : 0;
            bool used[256] = {false};
            for (int j = 0; j < B; ++j) used[loops[j % nloops]] = true;
            pa.nloops = 0;
            for (int r = 0; r < R; ++r)
                if (used[r]) pa.loop[pa.nloops++] = static_cast<uint8_t>(r);
        }
        const ripe::SeqGeom s = ripe::seq_geom(T, pa);
        for (int lt = 0; lt < s.total; ++lt) {
            const ripe::Tile t = ripe::tile_at(s, lt, pa);
            std::printf("%d %d %d %d %d\n", t.kind, t.t0, t.cnt, t.y, t.plane);
        }
        std::printf("E %d\n", s.total);
    }
    return 0;
}
