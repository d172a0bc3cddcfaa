"""Summaries of ncu CSV captures for the files under profiles/.

    # launch list (ncu --metrics gpu__time_duration.sum --csv ...) -> markdown table
    python -m gated_linear_attention_fwd_b200.profile_summary launches CSV --title T --command C > profiles/X.md

    # DRAM bytes of one op call (ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum --csv ...)
    # -> per-call traffic of the op, recorded in profiles/ncu_traffic.json with the hash of the
    #    op's sources (bench.py uses it only while the sources are unchanged)
    python -m gated_linear_attention_fwd_b200.profile_summary traffic CSV [CSV ...] --op fwd --calls N --workload W --command C
    #    (several CSVs: one capture per scan order, each of N calls; the figure is their mean)

Reads only the CSVs it is given; runs nothing.
"""
import argparse
import collections
import csv
import json
import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rows(path):
    rows = list(csv.reader(open(path)))
    for i, r in enumerate(rows):
        if r and r[0] == "ID":
            hdr = rows[i]
            return hdr, [dict(zip(hdr, x)) for x in rows[i + 1:] if len(x) == len(hdr)]
    raise SystemExit("no ncu CSV header in %s" % path)


def _short(name):
    """Kernel name without template arguments and parameter list."""
    name = re.sub(r"^void\s+", "", name)
    out, depth = "", 0
    for ch in name:
        if ch in "<(":
            if depth == 0 and ch == "(":
                break
            depth += 1
        elif ch in ">)":
            depth -= 1
        elif depth == 0:
            out += ch
    return out.strip().replace("::::", "::")  # an anonymous namespace leaves an empty component


def _value(r):
    v = float(r["Metric Value"].replace(",", ""))
    unit = r.get("Metric Unit", "")
    scale = {"ns": 1, "us": 1e3, "usecond": 1e3, "ms": 1e6, "msecond": 1e6, "nsecond": 1,
             "byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(unit, 1)
    return v * scale


def launches(args):
    _, rows = _rows(args.csv)
    tot = collections.OrderedDict()
    cnt = collections.Counter()
    for r in rows:
        if r["Metric Name"] != "gpu__time_duration.sum":
            continue
        k = _short(r["Kernel Name"])
        tot[k] = tot.get(k, 0.0) + _value(r)
        cnt[k] += 1
    allt = sum(tot.values())
    print("# %s\n" % args.title)
    print("Command (on one B200, after the same command exited 0 without ncu):\n")
    print("    " + args.command + "\n")
    print("ncu serialises launches and runs them with cold caches, so per-launch times are not bench")
    print("numbers; the shares are what should agree with the bench.\n")
    print("| kernel | launches | total (ns) | mean (ns) | share |")
    print("|---|---|---|---|---|")
    for k, t in sorted(tot.items(), key=lambda kv: -kv[1]):
        print("| %s | %d | %s | %s | %.1f%% |" % (k, cnt[k], format(int(t), ","), format(int(t / cnt[k]), ","),
                                                 100 * t / allt))


def traffic(args):
    sys.path.insert(0, ROOT)
    import bench  # noqa: E402  (source lists and hash of the ops)
    kernels = bench.OP_KERNELS[args.op]
    # an entry "a | b" names the kernel that replaces the other in some scan orders
    names = {n.strip() for k in kernels for n in k.split("|")}
    rows = [r for c in args.csv for r in _rows(c)[1]]
    calls = args.calls * len(args.csv)  # one capture per scan order, each of args.calls calls
    rd = wr = 0.0
    for r in rows:
        if _short(r["Kernel Name"]).split("::")[-1] not in names:
            continue
        if r["Metric Name"] == "dram__bytes_read.sum":
            rd += _value(r)
        elif r["Metric Name"] == "dram__bytes_write.sum":
            wr += _value(r)
    name = bench.OP_NAMES[args.op]
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    d = json.load(open(path)) if os.path.exists(path) else {}
    d = {k: v for k, v in d.items() if k in bench.OP_NAMES.values()}
    d[name] = {
        "source_sha": bench._src_hash(bench.OP_SOURCES[args.op]),
        "dram_bytes_per_call": int((rd + wr) / calls),
        "dram_read_bytes_per_call": int(rd / calls),
        "dram_write_bytes_per_call": int(wr / calls),
        "kernels": kernels,
        "workload": args.workload,
        "command": args.command,
    }
    with open(path, "w") as f:
        json.dump(d, f, indent=1)
        f.write("\n")
    print(json.dumps(d[name], indent=1))


def bench_ops():
    sys.path.insert(0, ROOT)
    import bench  # noqa: E402
    return bench.OP_NAMES.keys()


def main():
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="cmd", required=True)
    a = sub.add_parser("launches")
    a.add_argument("csv")
    a.add_argument("--title", required=True)
    a.add_argument("--command", required=True)
    t = sub.add_parser("traffic")
    t.add_argument("csv", nargs="+", help="one capture per scan order; the figure is their mean per call")
    t.add_argument("--op", choices=sorted(bench_ops()), required=True)
    t.add_argument("--calls", type=int, required=True)
    t.add_argument("--workload", required=True)
    t.add_argument("--command", required=True)
    args = ap.parse_args()
    {"launches": launches, "traffic": traffic}[args.cmd](args)


if __name__ == "__main__":
    main()
