"""Parity metrics between the CUDA engine and the fp64 oracle.

Tolerances (fixed by the engine's accuracy contract):
  per-layer hidden state      relative L2 <= 1e-2
  DeltaNet recurrent state    relative L2 <= 1e-3
  logits                      max |gpu - oracle| <= 2e-2 * std(oracle logits)
  greedy top-1 agreement      >= 99 %, a disagreement counting as a tie when
                              the oracle's top-1/top-2 margin is below twice
                              the step's measured logits error
"""
import numpy as np

HIDDEN_REL_L2 = 1e-2
STATE_REL_L2 = 1e-3
LOGITS_STD_FRAC = 2e-2
TOP1_AGREEMENT = 0.99


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def logits_err(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(gpu - ref).max()), LOGITS_STD_FRAC * float(ref.std())


def mean_kl(ref, gpu):
    """KL(softmax(ref) || softmax(gpu)) in nats."""
    ref = np.asarray(ref, np.float64)
    gpu = np.asarray(gpu, np.float64)
    lp = ref - ref.max()
    lp -= np.log(np.exp(lp).sum())
    lq = gpu - gpu.max()
    lq -= np.log(np.exp(lq).sum())
    return float((np.exp(lp) * (lp - lq)).sum())


class Tracker:
    """Accumulates per-step comparisons and asserts the contract."""

    def __init__(self):
        self.steps = 0
        self.agree_raw = 0
        self.agree_tie = 0
        self.worst_logit_ratio = 0.0
        self.worst_hidden = 0.0
        self.kl = []

    def logits(self, gpu, ref):
        err, tol = logits_err(gpu, ref)
        assert err <= tol, "logits max-abs %.3e > %.3e" % (err, tol)
        self.worst_logit_ratio = max(self.worst_logit_ratio, err / tol)
        g, r = int(np.argmax(gpu)), int(np.argmax(ref))
        self.steps += 1
        if g == r:
            self.agree_raw += 1
            self.agree_tie += 1
        elif ref[r] - ref[g] < 2 * err:
            self.agree_tie += 1
        self.kl.append(mean_kl(ref, gpu))

    def hidden(self, gpu, ref):
        for l in range(ref.shape[0]):
            e = rel_l2(gpu[l], ref[l])
            assert e <= HIDDEN_REL_L2, "layer %d hidden rel-L2 %.3e" % (l, e)
            self.worst_hidden = max(self.worst_hidden, e)

    def finish(self):
        assert self.steps > 0
        rate = self.agree_tie / self.steps
        assert rate >= TOP1_AGREEMENT, "top-1 agreement %.3f" % rate
        return {"steps": self.steps, "top1_raw": self.agree_raw / self.steps,
                "top1_tie_adjusted": rate, "worst_logit_err_over_tol": self.worst_logit_ratio,
                "worst_hidden_rel_l2": self.worst_hidden,
                "mean_kl_nats": float(np.mean(self.kl))}
