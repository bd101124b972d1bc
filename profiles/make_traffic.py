"""Write profiles/traffic.json: per-launch DRAM bytes (read + write) of the
benchmark's roofline kernels, from ncu captures of reduced cases scaled by
the units processed, with a hash of the kernel sources at capture time (the
benchmark reports null once a source changes).

  python profiles/make_traffic.py <kernel> <workload> <read_bytes> <write_bytes> <scale> <src>...
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
path = os.path.join(ROOT, "profiles", "traffic.json")
kernel, workload, rd, wr, scale = sys.argv[1:6]
srcs = sys.argv[6:]
h = hashlib.sha256()
for f in srcs:
    h.update(open(os.path.join(ROOT, f), "rb").read())
d = json.load(open(path)) if os.path.exists(path) else {}
d[kernel] = {"workload": workload, "bytes_per_launch": (float(rd) + float(wr)) * float(scale),
             "captured_read_bytes": float(rd), "captured_write_bytes": float(wr),
             "scale": float(scale), "sources": srcs, "sha256": h.hexdigest()}
json.dump(d, open(path, "w"), indent=1)
print(kernel, d[kernel]["bytes_per_launch"])
