"""Counts of mask rows that differ from the oracle's, collected by the GPU tests and
printed in pytest's terminal summary (spec rule: such rows are reported).

Each record: (what, rows differing, rows marginal, rows compared)."""
RECORDS = []


def record(what, differ, marginal, rows):
    RECORDS.append((what, int(differ), int(marginal), int(rows)))
