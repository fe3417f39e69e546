"""Write ``oracle/lloydmax_tables.json`` by calling only ``oracle.lloydmax``.

Run from the repository root:  python -m oracle.gen_tables
"""
import json
import os

from oracle import lloydmax


def main():
    tab = lloydmax.build_tables()
    path = os.path.join(os.path.dirname(lloydmax.__file__), "lloydmax_tables.json")
    with open(path, "w") as f:
        json.dump(tab, f, indent=1)
        f.write("\n")
    for b in range(1, lloydmax.B_MAX + 1):
        print(b, repr(tab["D"][b]))


if __name__ == "__main__":
    main()
