"""Markdown table of the parity reports a GPU test run logged.

    ANCHORKV_PARITY_LOG=parity.jsonl python -m pytest tests -m gpu
    python tests/parity_table.py parity.jsonl

Each line of the log is one compress parity case (tests/parity.py
`log_report`): the near-tie counts of every exact decision, the largest
relative errors of the continuous outputs, the fp64-refined rows and whether
the layout bytes matched the oracle's; or a tensor-core accumulation report.
"""
import json
import sys

COLS = ["near_tie_scored", "near_tie_slot", "near_tie_gamma", "near_tie_select", "near_tie_code", "exact_ties_slot",
        "max_rel_pooled", "max_rel_util", "refined_rows", "bytes_identical"]


def _cell(v) -> str:
    return "%.2e" % v if isinstance(v, float) else str(v)


def table(rows) -> str:
    out = ["| case | " + " | ".join(c.replace("near_tie_", "near-tie ").replace("_", " ") for c in COLS) + " |",
           "|---|" + "---:|" * len(COLS)]
    for r in rows:
        if "near_ties" in r:
            out.append(f"| {r['case']} | " + " | ".join(_cell(r.get(c, "")) for c in COLS) + " |")
    for r in rows:
        if "max_rel_acc_err" in r:
            out.append(f"\n{r['case']}: max |acc - <x,a>| / (||x|| ||a||) = {r['max_rel_acc_err']:.3e} "
                       f"over {r['pairs']} pairs")
    return "\n".join(out)


if __name__ == "__main__":
    with open(sys.argv[1]) as f:
        print(table([json.loads(line) for line in f if line.strip()]))
