"""The paged-prefill kernel's hand-over protocol, checked on a randomised
model (tests/prefill_protocol_model.py): every run ends, no mbarrier wait sees
a phase early, and every tensor-core product finds its operands in place --
for query-tile pairs whose KV walks have equal and different lengths, and for
one query tile only; with and without the converter role that rewrites bf16
V tiles as fp16 before the PV products read them."""
import pytest

from prefill_protocol_model import run

SHAPES = [(1, 1), (1, 2), (2, 2), (3, 4), (7, 8), (12, 12), (5, 0), (2, 0), (20, 21)]


@pytest.mark.parametrize("convert", [False, True])
@pytest.mark.parametrize("nt_a,nt_b", SHAPES)
def test_protocol_runs_clean(nt_a, nt_b, convert):
    for seed in range(12):
        run(nt_a, nt_b, seed, convert=convert)


PLANTED = {
    # QK(j) without waiting for PV(j-2): the product overwrites a P still being read
    "no_pv_wait": ('            if j >= 2:\n                yield from wait(f"o_done{w}{j & 1}", (j - 2) >> 1)\n', ""),
    # one P hand-over barrier instead of one per tile parity
    "single_p_full": ('bars[f"p_full{w}{j & 1}"].arrive()', 'bars[f"p_full{w}0"].arrive()'),
    # QK(j) waits for PV(j-1) on the other parity's barrier
    "wrong_pv_phase": ('yield from wait(f"o_done{w}{j & 1}", (j - 2) >> 1)',
                       'yield from wait(f"o_done{w}{(j - 1) & 1}", (j - 1) >> 1)'),
    # bf16 caches: PV waits for the landed V tile instead of the converted one
    "pv_before_conversion": ('                yield from wait(f"v_conv{j % vs}", j // vs)\n',
                             '                yield from wait(f"v_full{j % vs}", j // vs)\n'),
}


@pytest.mark.parametrize("mistake", sorted(PLANTED))
def test_model_catches_planted_mistakes(mistake):
    """Each planted protocol mistake must fail the model (overwritten operand,
    parity aliasing or deadlock) for some of the seeds."""
    import prefill_protocol_model as m
    src = open(m.__file__).read()
    old, new = PLANTED[mistake]
    assert src.count(old) == 1
    ns = {}
    exec(compile(src.replace(old, new), "planted", "exec"), ns)
    caught = 0
    for seed in range(20):
        try:
            ns["run"](6, 7, seed, max_steps=60000, convert=mistake == "pv_before_conversion")
        except AssertionError:
            caught += 1
    assert caught > 0
