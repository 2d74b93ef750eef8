"""The bench line's `gpu_launches` claim: the per-step launch counts bench.py derives from the
library's launch decisions, against the launch lists ncu recorded for the same workloads
(profiles/launches_480p5s_forward.md, launches_480p20s_stream.md, launches_480p5s_backward.md).
CPU only: nothing is launched here."""
import bench
from hybrid_softmax_linear_chunked_b200 import configs as C


def test_forward_480p5s_matches_launch_list():
    # ncu launch list of the 480x832 5 s forward: fold, scan, phi_q, attention, lone-tile
    # combine per step
    assert bench.forward_launches(C.WAN_480P_5S) == 5


def test_streaming_480p20s_matches_launch_list():
    # ncu launch list of the 20 s streaming step: six launches per call (S^T copy, phi_q,
    # attention, fold, lone-tile combine, state add with the next carry); the first call reads
    # no state, so it has no phi_q
    w = C.WAN_480P_20S_STREAM
    sched = bench.parse_schedule(None, w)
    bounds = bench.sched_bounds(sched)
    cap = max(ov for _, ov in sched)
    per_call = [bench.stream_call_launches(w.frame_tokens, s, e, ov, nxt, cap)
                for (_, s, e, ov, nxt) in bounds]
    assert len(per_call) == 27
    assert per_call[0] == 5 and set(per_call[1:]) == {6}


def test_backward_480p5s_matches_launch_list():
    # ncu launch list of one 480x832 5 s backward pass: 73 launches
    assert bench.backward_launches(C.WAN_480P_5S) == 73


def test_launch_rules_on_edge_schedules():
    # one query tile per chunk, its window one key tile: a lone tile, not split (no combine);
    # two query tiles per chunk: no lone tile
    assert bench.lone_parts(128, 1, 0, 0, 4, 4) == 1
    assert bench.lone_parts(256, 1, 0, 0, 4, 4) == 1
    # three query tiles over a three-tile window: the lone tile runs as 3 parts
    assert bench.lone_parts(384, 1, 0, 0, 1, 1) == 3
    # one chunk covering the 21 frames (256 query tiles): no fold, no phi_q, no combine
    assert bench.forward_launches(C.ablation(21, 1, 2)) == 2
    # the whole sequence as one context-parallel segment: the forward plus the segment sum
    w = C.WAN_480P_5S
    assert bench.segment_launches(w, 0, w.n_chunks) == bench.forward_launches(w) + 1
    # a 1-frame chunk (13 query tiles) after 3 frames, overlap 2, next overlap 1, carry 2: S^T
    # copy, phi_q, attention, fold of 2 frames, combine, then the state add and two carry
    # gathers (the chunk is shorter than the carry)
    assert bench.stream_call_launches(1560, 3, 4, 2, 1, 2) == 8
