"""The scheduling-overhead decoder on hand-made traces (no GPU): every
number below is worked out by hand from the definition
overhead = t_start - max(fire(dep), end of the previous task on the SM)."""
import numpy as np

from persistent_decode_megakernel_02_b200 import trace as tr

DT = np.dtype([("t_ready", np.uint64), ("t_start", np.uint64), ("t_input", np.uint64),
               ("t_done", np.uint64), ("t_end", np.uint64), ("t_wait", np.uint64),
               ("sm", np.int32), ("kind", np.int32), ("layer", np.int32), ("trig_event", np.int32)])


def _graph():
    # task: kind, layer, dep, trig, begin, end, sm, slot
    tasks = np.array([
        [0, 0, -1, 0, 0, 1, 0, 0],   # 0: QKV on SM 0
        [0, 0, -1, 0, 1, 2, 1, 1],   # 1: QKV on SM 1
        [1, 0, 0, 1, 0, 1, 0, 0],    # 2: attention on SM 0, waits on event 0
        [1, 0, 0, 1, 1, 2, 1, 1],    # 3: attention on SM 1
        [2, 0, 1, 2, 0, 1, 0, 0],    # 4: O-proj on SM 0, waits on event 1
    ], np.int32)
    queue = np.array([0, 2, 4, 1, 3], np.int32)
    qoff = np.array([0, 3, 5], np.int32)
    t = np.zeros(5, DT)
    t["t_start"] = [100, 110, 300, 260, 700]
    t["t_end"] = [200, 250, 400, 600, 800]
    return t, tasks, queue, qoff


def test_overhead_is_start_minus_the_later_of_dependency_fire_and_previous_end():
    t, tasks, queue, qoff = _graph()
    d = tr.task_overheads(t, tasks, queue, qoff)
    # event 0 fires at 250 (last QKV end), event 1 at 600 (last attention end)
    assert np.isnan(d["fire_dep"][0]) and np.isnan(d["fire_dep"][1])
    assert d["fire_dep"][2] == 250 and d["fire_dep"][3] == 250 and d["fire_dep"][4] == 600
    # previous task on the same SM
    assert np.isnan(d["prev_end"][0]) and np.isnan(d["prev_end"][1])
    assert d["prev_end"][2] == 200 and d["prev_end"][3] == 250 and d["prev_end"][4] == 400
    # task 2: ready at max(250, 200) = 250, started 300 -> 50 ns
    # task 3: ready at max(250, 250) = 250, started 260 -> 10 ns
    # task 4: ready at max(600, 400) = 600, started 700 -> 100 ns
    # tasks 0, 1: nothing to wait for -> undefined
    ov = d["overhead"]
    assert np.isnan(ov[0]) and np.isnan(ov[1])
    assert list(ov[2:]) == [50.0, 10.0, 100.0]


def test_summary_reports_per_kind_statistics_in_microseconds():
    t, tasks, queue, qoff = _graph()
    d = tr.task_overheads(t, tasks, queue, qoff)
    s = tr.summarize(d["overhead"], d["kind"])
    assert s["all"]["n"] == 3
    assert abs(s["all"]["median_us"] - 0.05) < 1e-12 and abs(s["all"]["max_us"] - 0.1) < 1e-12
    assert s["attn"]["n"] == 2 and abs(s["attn"]["mean_us"] - 0.03) < 1e-12
    assert s["oproj"]["n"] == 1 and abs(s["oproj"]["median_us"] - 0.1) < 1e-12
    assert s["qkv"]["n"] == 0


def test_a_task_that_starts_before_its_event_fires_shows_a_negative_overhead():
    # tagged waits: an attention task needs only its own heads' words and may
    # start before the last QKV task of the op has posted
    t, tasks, queue, qoff = _graph()
    t["t_start"][3] = 240
    t["t_end"][1] = 230      # SM 1's previous task ended at 230
    t["t_end"][0] = 250      # event 0 now fires at 250 (task 0)
    d = tr.task_overheads(t, tasks, queue, qoff)
    assert d["overhead"][3] == 240 - 250


def test_critical_path_increments_and_transitions_by_hand():
    t, tasks, queue, qoff = _graph()
    t["t_ready"] = [100, 110, 290, 255, 690]
    t["t_input"] = [120, 130, 310, 270, 720]
    t["t_done"] = [190, 240, 390, 580, 790]
    # layers=[0]: every op of layer 0 after the first counts
    cp = tr.critical_path(t, tasks, layers=[0])
    # QKV last done 240; attention last done 580 -> 340, last ready 290 -> 50;
    # O-proj done 790 -> 210 after 580, ready 690 -> 110
    assert cp["attn"] == {"inc_us": 0.34, "to_ready_us": 0.05, "n": 1}
    assert cp["oproj"] == {"inc_us": 0.21, "to_ready_us": 0.11, "n": 1}
    assert "qkv" not in cp
    tv = tr.transitions(t, tasks)
    # SM 0: 0 -> 2: tail 200-190 = 10, to_ready 290-200 = 90, compute 390-310 = 80
    #        2 -> 4: tail 400-390 = 10, to_ready 690-400 = 290, compute 790-720 = 70
    # SM 1: 1 -> 3: tail 250-240 = 10, to_ready 255-250 = 5, compute 580-270 = 310
    assert tv["oproj"]["to_ready_us"] == 0.29 and tv["oproj"]["compute_us"] == 0.07
    a = tv["attn"]     # medians of (90, 5) and (80, 310)
    assert a["n"] == 2 and abs(a["to_ready_us"] - 0.0475) < 1e-12 and abs(a["compute_us"] - 0.195) < 1e-12
    assert a["tail_us"] == 0.01
