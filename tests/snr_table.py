"""Prints the routing failure rate against Phi(-SNR) for the pages' setting
(d = 64, B in {128, 256, 512}) through the oracle router; the same harness
as tests/test_snr_recall.py.  Usage: python tests/snr_table.py [n_seq]"""
import math
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from tests.test_snr_recall import D, _delta_for, _oracle_trials  # noqa: E402
from oracle import moba_oracle as O  # noqa: E402


def main():
    n_seq = int(sys.argv[1]) if len(sys.argv) > 1 else 250
    h = 4
    print("| B | SNR | delta_mu_eff | Phi(-SNR) | empirical | trials | 1-sigma |")
    print("|---:|---:|---:|---:|---:|---:|---:|")
    for B in (128, 256, 512):
        for snr in (0.5, 1.0, 1.5, 2.0):
            fails, _ = _oracle_trials(B, snr, n_seq, h)
            p = O.router_p_fail(snr)
            print("| %d | %.1f | %.3f | %.4f | %.4f | %d | %.4f |" % (
                B, snr, _delta_for(snr, B), p, fails.mean(), len(fails), math.sqrt(p * (1 - p) / len(fails))))


if __name__ == "__main__":
    main()
