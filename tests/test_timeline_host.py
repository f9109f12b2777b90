"""Host side of the kernels' timeline: timeline_summary on hand-built records
(no GPU needed).  The records are what timeline_stop decodes from the
device buffer: kind, role, CTA, sub, id and two %globaltimer stamps in ns."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import mixture_experts_expert_softmax_b200 as moe  # noqa: E402


def _rec(kind, role, cta, ident, t0_us, t1_us, sub=0):
    return {"kind": kind, "role": role, "cta": cta, "sub": sub, "id": ident,
            "t0": int(t0_us * 1000) + 10**12, "t1": int(t1_us * 1000) + 10**12}


def test_summary_counts_durations_and_spans():
    recs = [_rec("small_t", "phase1", c, c, 0.0, 10.0 + c) for c in range(3)]
    recs += [_rec("small_t", "barrier", c, c, 10.0 + c, 13.0) for c in range(3)]
    s = moe.timeline_summary(recs)
    assert s["small_t/phase1"] == {"n": 3, "mean_us": 11.0, "max_us": 12.0, "span_us": 12.0}
    assert s["small_t/barrier"] == {"n": 3, "mean_us": 2.0, "max_us": 3.0, "span_us": 3.0}


def test_summary_mma_bins_busy_and_gaps():
    # two CTAs; CTA 0 runs tiles back to back with a 0.5 us gap, CTA 1 one
    # tile that starts 12 us after the first MMA
    recs = [_rec("gemm_fused", "mma", 0, 0, 0.0, 4.0),
            _rec("gemm_fused", "mma", 0, 2, 4.5, 8.5),
            _rec("gemm_fused", "mma", 1, 1, 12.0, 18.0),
            _rec("gemm_fused", "epilogue", 0, 0, 4.0, 5.0)]
    s = moe.timeline_summary(recs)
    m = s["gemm_fused/mma"]
    assert m["n"] == 3 and m["max_us"] == 6.0 and m["span_us"] == 18.0
    # bins of 10 us by start: tiles at 0 and 4.5 us, then the one at 12 us
    assert m["by_start_10us"] == {0: [2, 4.0], 10: [1, 6.0]}
    assert m["cta_mma_us_min_med_max"] == [6.0, 8.0, 8.0]
    assert m["tile_gap_us_median"] == 0.5
    # other roles get the plain statistics only
    assert set(s["gemm_fused/epilogue"]) == {"n", "mean_us", "max_us", "span_us"}


def test_summary_of_nothing_is_empty():
    assert moe.timeline_summary([]) == {}


def test_decoder_names_match_the_device_codes():
    """The kind and role codes the kernels write (an enum in the device
    header) decode to the names timeline_stop reports."""
    import re
    src = open(os.path.join(ROOT, "mixture_experts_expert_softmax_b200", "csrc",
                            "common.cuh")).read()
    codes = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(kTl\w+)\s*=\s*(\d+)", src)}
    kinds = {"kTlGemm1": "gemm1", "kTlGemm2": "gemm2", "kTlFused": "gemm_fused",
             "kTlSmallT": "small_t"}
    roles = {"kTlProducer": "producer", "kTlMma": "mma", "kTlEpilogue": "epilogue",
             "kTlPhase1": "phase1", "kTlBarrier": "barrier", "kTlActLoad": "act_load",
             "kTlW2Wait": "w2_wait", "kTlPhase2": "phase2", "kTlItems": "phase2_dots"}
    assert set(kinds) | set(roles) <= set(codes)
    assert {codes[c]: n for c, n in kinds.items()} == moe.TIMELINE_KINDS
    assert {codes[c]: n for c, n in roles.items()} == moe.TIMELINE_ROLES
