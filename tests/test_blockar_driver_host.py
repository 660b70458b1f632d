"""Host control of the block-AR driver (generate_blocks) on CPU, against a
stand-in context that records the calls: one causal prefill, up to
max_steps steps per block ending at the first step whose all-settled (or
adaptive-stop) flags are set for every sequence, K - 1 commits (K with
commit_last), the threshold schedule evaluated per step, and the entropy
path's temperatures and previous-argmax chaining."""
import torch

import block_discrete_diffusion_denoise_b200 as dgp


class FakeCtx:
    """Denoising step: out = in + 1; sequence b settles from step settle_at[b] on."""

    def __init__(self, settle_at, canvas=8):
        self.cfg = {"canvas": canvas}
        self.settle_at = settle_at
        self.calls = []

    def prefill(self, prefix):
        self.calls.append(("prefill", int(prefix.shape[1])))

    def _step(self, cin, step, cout, flags):
        cout.copy_(cin + 1)
        for b, s0 in enumerate(self.settle_at):
            flags[b] = 1 if step >= s0 else 0

    def denoise_step(self, cin, step, seed, tau, cout, conf=None, settled=None):
        self.calls.append(("step", step, float(tau)))
        conf.fill_(0.5)
        self._step(cin, step, cout, settled)

    def denoise_step_entropy(self, cin, step, seed, temperature, gamma, stop_entropy, cout, prev_argmax=None,
                             argmax_out=None, entropy=None, stopped=None):
        self.calls.append(("entropy", step, round(float(temperature), 6), prev_argmax is None,
                           argmax_out.data_ptr() if argmax_out is not None else None))
        entropy.fill_(0.1)
        argmax_out.copy_(cin)
        self._step(cin, step, cout, stopped)

    def sync(self):
        pass

    def commit_block(self, block):
        self.calls.append(("commit", int(block[0, 0])))


def _init(k):
    return torch.full((2, 8), 100 * k, dtype=torch.int32)


def test_threshold_path_stops_at_the_first_all_settled_step_and_commits_k_minus_one_blocks():
    ctx = FakeCtx(settle_at=[2, 4])                      # sequence 1 settles later: the batch waits for it
    out = dgp.generate_blocks(ctx, torch.zeros(2, 5, dtype=torch.int32), _init, n_blocks=3, max_steps=10,
                              tau=lambda s: 0.9 - 0.1 * s, seed=7)
    assert out["steps"] == [5, 5, 5] and out["settled"] == [True] * 3
    for k in range(3):
        assert torch.equal(out["blocks"][k], _init(k) + 5)
    kinds = [c[0] for c in ctx.calls]
    assert kinds[0] == "prefill" and ctx.calls[0][1] == 5
    assert kinds.count("commit") == 2 and kinds[-1] == "step"        # the last block is not committed
    taus = [c[2] for c in ctx.calls if c[0] == "step"][:5]
    assert all(abs(a - (0.9 - 0.1 * s)) < 1e-6 for s, a in enumerate(taus))   # tau(s) evaluated per step
    commits = [c[1] for c in ctx.calls if c[0] == "commit"]
    assert commits == [0 + 5, 100 + 5]                    # each block's final canvas is what gets committed


def test_commit_last_and_the_step_cap():
    ctx = FakeCtx(settle_at=[99, 99])                     # never settles: every block runs max_steps
    out = dgp.generate_blocks(ctx, torch.zeros(2, 3, dtype=torch.int32), _init, n_blocks=2, max_steps=4, tau=0.5,
                              seed=1, commit_last=True)
    assert out["steps"] == [4, 4] and out["settled"] == [False, False]
    assert [c[0] for c in ctx.calls].count("commit") == 2


def test_entropy_path_anneals_the_temperature_and_chains_the_argmax():
    ctx = FakeCtx(settle_at=[3, 3])
    out = dgp.generate_blocks(ctx, torch.zeros(2, 3, dtype=torch.int32), _init, n_blocks=1, max_steps=48, tau=None,
                              seed=1, entropy={"gamma": 2.0, "stop_entropy": 0.5})
    assert out["steps"] == [4] and out["settled"] == [True]
    ent = [c for c in ctx.calls if c[0] == "entropy"]
    assert [c[1] for c in ent] == [0, 1, 2, 3]
    assert [c[2] for c in ent] == [round(dgp.anneal_temperature(s, 48), 6) for s in range(4)]
    assert ent[0][3] is True and all(c[3] is False for c in ent[1:])   # no previous argmax at a block's first step
    assert len({c[4] for c in ent}) == 1                               # one argmax buffer, passed back each step
    assert abs(dgp.anneal_temperature(0, 48) - 0.8) < 1e-12 and abs(dgp.anneal_temperature(47, 48) - 0.4) < 1e-12
